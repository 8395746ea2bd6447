"""Generate ``winograd_gen.cuh``: straight-line Winograd F(m x m, 3 x 3) transforms.

The matrices are derived here, exactly, in rational arithmetic, by the
Cook-Toom / Lavin-Gray construction ("Fast Algorithms for Convolutional Neural
Networks", Lavin and Gray, 2016): for a polynomial product of a length-3
filter and a length-m signal evaluated at the alpha = m + 2 points
p_0..p_{alpha-2} and infinity,

  * A^T (m x alpha):  A^T[i][j] = p_j^i;  the infinity column is e_{m-1};
  * G (alpha x 3):    G[j][k]   = p_j^k;  the infinity row is e_2;
  * B^T (alpha x alpha) = (V^{-1})^T where V[j][n] = p_j^n (infinity row e_{alpha-1});

the transposition principle turns that product into the correlation
y_i = sum_k g_k d_{i+k} = A^T[(G g) . (B^T d)].  Row j of B^T is then scaled by
f_j = prod_{l != j}(p_j - p_l) (and row j of G by 1/f_j), which makes B^T
small rationals, and rows are sign-normalised so B^T's first non-zero entry is
positive.  The 2D transforms are the 1D ones applied to rows and columns.

Points: F(2,3) {0, 1, -1}; F(4,3) {0, 1, -1, 2, -2}; F(6,3) {0, +-1, +-2, +-1/2}.

Run ``python gen_winograd.py`` to rewrite the header; the test suite checks
that the committed header matches and that the matrices reproduce direct
correlation exactly.
"""
from fractions import Fraction as Fr
import os
import sys

POINTS = {
    2: [Fr(0), Fr(1), Fr(-1)],
    4: [Fr(0), Fr(1), Fr(-1), Fr(2), Fr(-2)],
    6: [Fr(0), Fr(1), Fr(-1), Fr(2), Fr(-2), Fr(1, 2), Fr(-1, 2)],
}
R = 3


def _inverse(M):
    n = len(M)
    A = [list(row) + [Fr(int(i == j)) for j in range(n)] for i, row in enumerate(M)]
    for c in range(n):
        p = next(r for r in range(c, n) if A[r][c] != 0)
        A[c], A[p] = A[p], A[c]
        pv = A[c][c]
        A[c] = [x / pv for x in A[c]]
        for r in range(n):
            if r != c and A[r][c] != 0:
                f = A[r][c]
                A[r] = [a - f * b for a, b in zip(A[r], A[c])]
    return [row[n:] for row in A]


def matrices(m):
    """Exact (AT, G, BT) for F(m, 3) as lists of Fractions."""
    pts = POINTS[m]
    a = m + R - 1
    AT = [[p ** i for p in pts] + [Fr(int(i == m - 1))] for i in range(m)]
    G = [[p ** k for k in range(R)] for p in pts] + [[Fr(int(k == R - 1)) for k in range(R)]]
    V = [[p ** n for n in range(a)] for p in pts] + [[Fr(int(n == a - 1)) for n in range(a)]]
    Vi = _inverse(V)
    BT = [[Vi[n][j] for n in range(a)] for j in range(a)]
    for j in range(a - 1):
        f = Fr(1)
        for l in range(a - 1):
            if l != j:
                f *= pts[j] - pts[l]
        BT[j] = [x * f for x in BT[j]]
        G[j] = [x / f for x in G[j]]
    for j in range(a):
        first = next(x for x in BT[j] if x != 0)
        if first < 0:
            BT[j] = [-x for x in BT[j]]
            G[j] = [-x for x in G[j]]
    return AT, G, BT


def _lit(q: Fr) -> str:
    """A float literal for q: exact when q is dyadic, else the nearest float."""
    import numpy as np
    v = np.float32(float(q))
    s = repr(float(v))
    if "e" not in s and "." not in s:
        s += ".0"
    return s + "f"


def _expr(row, src, pick=None):
    """Sum of row[k] * src[k] as C; pick limits the terms to a parity (0/1)."""
    terms = []
    for k, c in enumerate(row):
        if c == 0 or (pick is not None and k % 2 != pick):
            continue
        if c == 1:
            terms.append(f"+ {src}[{k}]")
        elif c == -1:
            terms.append(f"- {src}[{k}]")
        elif c > 0:
            terms.append(f"+ {_lit(c)} * {src}[{k}]")
        else:
            terms.append(f"- {_lit(-c)} * {src}[{k}]")
    if not terms:
        return "0.0f"
    s = " ".join(terms)
    return s[2:] if s.startswith("+ ") else "-" + s[2:]


def _row_pairs(M):
    """Pairs (p, q, s_even, s_odd) with M[q][n] = s_even*M[p][n] for even n and
    s_odd*M[p][n] for odd n, s_even = -s_odd: rows of a +-a point pair."""
    used, pairs = set(), []
    for p in range(len(M)):
        if p in used:
            continue
        for q in range(p + 1, len(M)):
            if q in used:
                continue
            for se in (1, -1):
                so = -se
                if all(M[q][n] == (se if n % 2 == 0 else so) * M[p][n] for n in range(len(M[p]))) and \
                        any(M[p][n] != 0 for n in range(0, len(M[p]), 2)) and \
                        any(M[p][n] != 0 for n in range(1, len(M[p]), 2)):
                    pairs.append((p, q, se, so))
                    used.update((p, q))
                    break
            if p in used:
                break
    return pairs


def _emit_rows(name, M, n_in):
    """y = M x with paired rows sharing their even / odd partial sums."""
    out = [f"__device__ __forceinline__ void {name}(const float* x, float* y) {{"]
    pairs = _row_pairs(M)
    done = set()
    for (p, q, se, so) in pairs:
        out.append(f"  {{ const float e = {_expr(M[p], 'x', 0)}, o = {_expr(M[p], 'x', 1)};")
        out.append(f"    y[{p}] = e + o;")
        out.append(f"    y[{q}] = {'' if se > 0 else '-'}e {'-' if se > 0 else '+'} o; }}")
        done.update((p, q))
    for r in range(len(M)):
        if r not in done:
            out.append(f"  y[{r}] = {_expr(M[r], 'x')};")
    out.append("}")
    return out


def _col_pairs(M):
    """Column pairs (p, q) with M[i][q] = M[i][p] for even i and -M[i][p] for odd i."""
    cols = len(M[0])
    used, pairs = set(), []
    for p in range(cols):
        if p in used:
            continue
        for q in range(p + 1, cols):
            if q in used:
                continue
            if all(M[i][q] == (1 if i % 2 == 0 else -1) * M[i][p] for i in range(len(M))) and \
                    any(M[i][p] != 0 for i in range(len(M))):
                pairs.append((p, q))
                used.update((p, q))
                break
    return pairs


def _emit_cols(name, M):
    """y = M x with paired columns combined first: s = x_p + x_q, d = x_p - x_q."""
    out = [f"__device__ __forceinline__ void {name}(const float* x, float* y) {{"]
    pairs = _col_pairs(M)
    paired = {}
    for k, (p, q) in enumerate(pairs):
        out.append(f"  const float s{k} = x[{p}] + x[{q}], d{k} = x[{p}] - x[{q}];")
        paired[p] = k
    lone = [c for c in range(len(M[0])) if all(c not in pq for pq in pairs)]
    for i, row in enumerate(M):
        terms = []
        for c in lone:
            if row[c] != 0:
                terms.append((row[c], f"x[{c}]"))
        for p, k in paired.items():
            if row[p] != 0:
                terms.append((row[p], f"{'s' if i % 2 == 0 else 'd'}{k}"))
        parts = []
        for c, v in terms:
            if c == 1:
                parts.append(f"+ {v}")
            elif c == -1:
                parts.append(f"- {v}")
            elif c > 0:
                parts.append(f"+ {_lit(c)} * {v}")
            else:
                parts.append(f"- {_lit(-c)} * {v}")
        e = " ".join(parts) if parts else "0.0f"
        e = e[2:] if e.startswith("+ ") else ("-" + e[2:] if e.startswith("- ") else e)
        out.append(f"  y[{i}] = {e};")
    out.append("}")
    return out


def emit() -> str:
    out = []
    out.append("// GENERATED by gen_winograd.py -- do not edit by hand.")
    out.append("// 1D Winograd F(m, 3) transforms, from the exact Cook-Toom matrices:")
    out.append("//   *_bt: y = B^T x (alpha -> alpha), *_g: y = G x (3 -> alpha), *_at: y = A^T x (alpha -> m).")
    out.append("// Rows (B^T, G) or columns (A^T) belonging to a +-a point pair share their")
    out.append("// even / odd partial sums, which halves the arithmetic.")
    out.append("#pragma once")
    out.append("")
    for m in sorted(POINTS):
        AT, G, BT = matrices(m)
        a = m + R - 1
        out.append(f"// F({m}x{m}, 3x3): alpha = {a}")
        out += _emit_rows(f"wino{m}_bt", BT, a)
        out += _emit_rows(f"wino{m}_g", G, R)
        out += _emit_cols(f"wino{m}_at", AT)
        out.append("")
    return "\n".join(out) + "\n"


HEADER = os.path.join(os.path.dirname(os.path.abspath(__file__)), "winograd_gen.cuh")

if __name__ == "__main__":
    text = emit()
    with open(HEADER, "w") as f:
        f.write(text)
    print(HEADER, file=sys.stderr)
