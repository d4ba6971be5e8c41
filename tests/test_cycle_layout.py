"""DraftCycle's I/O arenas (host logic, no GPU): every tensor of a step's
inputs (and of its results) is a view into one byte buffer, at a 256-byte
aligned offset, with its own shape and dtype, and no two views overlap -- so
one copy moves a whole step's inputs and one its results."""
import torch

from block_draft_selection_b200.cycle import _arena, _nbytes, io_layout


def test_arena_views_are_aligned_disjoint_and_typed():
    specs = [("H", (7, 2560), torch.bfloat16), ("x", (1, 8, 2560), torch.bfloat16), ("prev", (1, 2560), torch.bfloat16),
             ("target", (1, 8), torch.int32), ("odd", (3,), torch.int32)]
    buf, views = _arena(specs, "cpu")
    assert buf.dtype == torch.uint8 and buf.dim() == 1
    spans = []
    for name, shape, dt in specs:
        v = views[name]
        assert tuple(v.shape) == shape and v.dtype == dt and v.is_contiguous()
        off = v.data_ptr() - buf.data_ptr()
        assert off % 256 == 0
        spans.append((off, off + v.numel() * v.element_size()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= buf.numel()
    # writes through a view land in the buffer
    views["target"].fill_(7)
    off = views["target"].data_ptr() - buf.data_ptr()
    assert buf[off:off + 32].view(torch.int32).tolist() == [7] * 8


def test_status_word_is_in_both_copies():
    """The status word closes the input span (so the host-to-device copy
    clears it every step) and opens the result span (so the device-to-host
    copy returns it); no input or result overlaps it or each other."""
    ins = [("H", (7, 2560), torch.bfloat16), ("x", (1, 8, 2560), torch.bfloat16), ("prev", (1, 2560), torch.bfloat16),
           ("target", (1, 8), torch.int32)]
    outs = [("path_tok", (1, 7), torch.int32), ("accept_len", (1,), torch.int32), ("next_token", (1,), torch.int32),
            ("y", (1, 8, 2560), torch.bfloat16)]
    offs, in_end, out_begin, end = io_layout(ins, outs)
    s = offs["status"][0]
    assert out_begin == s and in_end == s + 4 and s % 256 == 0
    size = lambda n: _nbytes(offs[n][1], offs[n][2])
    for n, _, _ in ins:
        assert offs[n][0] + size(n) <= s
    for n, _, _ in outs:
        assert offs[n][0] >= s + 4 and offs[n][0] + size(n) <= end
    spans = sorted((offs[n][0], offs[n][0] + size(n)) for n in offs)
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
