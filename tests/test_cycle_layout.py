"""DraftCycle's I/O arenas (host logic, no GPU): every tensor of a step's
inputs (and of its results) is a view into one byte buffer, at a 256-byte
aligned offset, with its own shape and dtype, and no two views overlap -- so
one copy moves a whole step's inputs and one its results."""
import torch

from block_draft_selection_b200.cycle import _arena


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
