"""Exact rational arithmetic on the stored bit patterns (test-side pins).

Independent of the oracle's numpy path: every value is a Fraction built from
the bf16 / fp32 bits, and every sum and product is exact."""
from fractions import Fraction

K = 16


def bf(b):
    """One bf16 bit pattern -> Fraction."""
    b = int(b)
    sign = -1 if b & 0x8000 else 1
    exp = (b >> 7) & 0xFF
    man = b & 0x7F
    if exp == 0:
        return sign * Fraction(man, 1 << 133)
    return sign * Fraction(128 + man, 128) * Fraction(2) ** (exp - 127)


def emb_rows(E, tokens):
    """{token: [Fraction] * r} for the listed tokens of the bf16 table E."""
    r = E.shape[1]
    return {int(c): [bf(E[int(c), s]) for s in range(r)] for c in set(int(t) for t in tokens)}


def mat(M):
    r = M.shape[0]
    return [[bf(M[s, t]) for t in range(r)] for s in range(r)]


def bilinear(ea, Mf, eb):
    """ea . M . eb, exactly."""
    r = len(Mf)
    u = [sum(ea[s] * Mf[s][t] for s in range(r)) for t in range(r)]
    return sum(u[t] * eb[t] for t in range(r))


def exact_pairs(logp, idx, E, M, b, L, K=K):
    """S_i[j][k] = lp_i(j) + lp_{i+1}(k) + e_{c_ij} M e_{c_{i+1,k}} for block b."""
    Mf = mat(M)
    rows = emb_rows(E, idx[b * L:(b + 1) * L].ravel())
    lp = [[Fraction(float(logp[b * L + i, j])) for j in range(K)] for i in range(L)]
    S = []
    for i in range(L - 1):
        Si = [[lp[i][j] + lp[i + 1][k] + bilinear(rows[int(idx[b * L + i, j])], Mf,
                                                  rows[int(idx[b * L + i + 1, k])])
               for k in range(K)] for j in range(K)]
        S.append(Si)
    return S


def exact_anchor(logp, idx, E, M, anchor, b, L, K=K):
    """S_a[k] = lp_0(k) + e_anchor M e_{c_0k} for block b."""
    Mf = mat(M)
    rows = emb_rows(E, list(idx[b * L].ravel()) + [int(anchor)])
    ea = rows[int(anchor)]
    return [Fraction(float(logp[b * L, k])) + bilinear(ea, Mf, rows[int(idx[b * L, k])]) for k in range(K)]
