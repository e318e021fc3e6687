"""Generate straight-line real-input FFT codelets for libkvq (kvq_rfft.cuh).

    python rotated_int4_kv_kvq_b200/csrc/gen_rfft.py

For n in {32, 64} it emits two-lane codelets over f2 values (two
independent transforms in lock step, one per lane of each packed fp32x2
register):

  rfft<n>x2_fwd(x, y):  y[0] = X_0/sqrt2, y[1] = X_{n/2}/sqrt2,
                        y[2k] = Re X_k, y[2k+1] = Im X_k   (1 <= k < n/2),
                        X_k = sum_m x_m exp(-2 pi i k m / n)  (unnormalized);
  rfft<n>x2_inv(y, x):  the transpose (adjoint) of the forward map,
                        x_m = (1/2) sum_k X_k exp(+2 pi i k m / n) with X
                        rebuilt from y in the same packing (X_0 = sqrt2 y[0],
                        X_{n/2} = sqrt2 y[1]), i.e. half the unnormalized
                        inverse real DFT.

The forward transform follows the split-radix decomposition for real data
(even samples through a half-length real DFT, samples 4m+1 and 4m+3
through two quarter-length real DFTs, recombined with twiddles W^k and
W^3k), keeping only the non-redundant half of every Hermitian spectrum; the
inverse is its transpose, built by reversing every edge of the forward
graph, so it costs the same number of operations.  The generator builds an
expression graph with hash-consing, folds trivial twiddles (+-1, +-i) and
negations into add/sub, writes a twiddle product in tangent form (c (x +
(s/c) y), or with the roles of c and s swapped) so that the common factor
is a multiply that can be carried: a sum of two such multiples keeps one
factor outside (one multiply-add), and a multiply whose consumers are all
adds is folded into them.  It checks the graph numerically against numpy's
FFT, then the emitted instruction list (with the polarity of every output,
see emit_x2) against the graph before writing anything.  Twiddle constants
are evaluated in double and rounded once to float.
"""

from __future__ import annotations

import math
import os
import sys

import numpy as np


class R:
    """A real value: `sign * node`, node None meaning exactly zero."""

    __slots__ = ("node", "sign")

    def __init__(self, node, sign=1):
        self.node = node
        self.sign = sign


ZERO = R(None, 1)


class Graph:
    def __init__(self):
        self.nodes = []  # (op, args)
        self.memo = {}

    def _mk(self, op, *args):
        key = (op, args)
        if key not in self.memo:
            self.memo[key] = len(self.nodes)
            self.nodes.append(key)
        return self.memo[key]

    def inp(self, name):
        return R(self._mk("in", name))

    @staticmethod
    def neg(a):
        return R(a.node, -a.sign)

    def add(self, a, b):
        if a.node is None:
            return b
        if b.node is None:
            return a
        if a.sign == b.sign:
            lo, hi = sorted((a.node, b.node))
            return R(self._mk("add", lo, hi), a.sign)
        if a.node == b.node:
            return ZERO
        pos, neg_ = (a, b) if a.sign > 0 else (b, a)
        return R(self._mk("sub", pos.node, neg_.node), 1)

    def sub(self, a, b):
        return self.add(a, self.neg(b))

    def mulc(self, a, c):
        if a.node is None or c == 0.0:
            return ZERO
        if c == 1.0:
            return a
        if c == -1.0:
            return self.neg(a)
        op, args = self.nodes[a.node]
        if op == "mul":  # (x m) c = x (m c): one multiply, not two
            x, m = args
            return self.mulc(R(x, a.sign), float(np.float32(m * c)))
        s = a.sign * (1 if c > 0 else -1)
        return R(self._mk("mul", a.node, abs(c)), s)

    def fmac(self, a, c, b):
        """a * c + b with c a constant (one fused multiply-add)."""
        if a.node is None or c == 0.0:
            return b
        if b.node is None:
            return self.mulc(a, c)
        if c in (1.0, -1.0):
            return self.add(self.mulc(a, c), b)
        cc = a.sign * b.sign * c
        return R(self._mk("fma", a.node, cc, b.node), b.sign)

    def split_mul(self, a):
        """a = m * x with x a node: (x, m); (a, None) when a is no multiple."""
        if a.node is None:
            return a, None
        op, args = self.nodes[a.node]
        if op == "mul":
            return R(args[0], a.sign), args[1]
        return a, None

    def add_common(self, a, b, sb=1):
        """a + sb * b; when both are constant multiples m_a x, m_b y, as
        m_a (x + sb (m_b / m_a) y): one multiply-add, the factor m_a left for
        the emitter to fold into the adds that consume the sum."""
        xa, ma = self.split_mul(a)
        xb, mb = self.split_mul(b)
        if ma is None or mb is None:
            return self.add(a, b) if sb > 0 else self.sub(a, b)
        r = float(np.float32(sb * mb / ma))
        return self.mulc(self.fmac(xb, r, xa), ma)

    def fmac_common(self, a, c, b):
        """c a + b; a constant factor of a is folded into c, and one of b is
        kept out (as for add_common)."""
        xa, ma = self.split_mul(a)
        xb, mb = self.split_mul(b)
        ca = c if ma is None else float(np.float32(c * ma))
        if mb is None:
            return self.fmac(xa, ca, b)
        return self.mulc(self.fmac(xa, float(np.float32(ca / mb)), xb), mb)

    def cadd_common(self, a, b):
        return (self.add_common(a[0], b[0]), self.add_common(a[1], b[1]))

    def csub_common(self, a, b):
        return (self.add_common(a[0], b[0], -1), self.add_common(a[1], b[1], -1))

    # complex helpers: values are (re, im) pairs of R
    def cadd(self, a, b):
        return (self.add(a[0], b[0]), self.add(a[1], b[1]))

    def csub(self, a, b):
        return (self.sub(a[0], b[0]), self.sub(a[1], b[1]))

    @staticmethod
    def conj(a):
        return (a[0], Graph.neg(a[1]))

    @staticmethod
    def mul_i(a):  # i * a
        return (Graph.neg(a[1]), a[0])

    @staticmethod
    def mul_mi(a):  # -i * a
        return (a[1], Graph.neg(a[0]))

    def ctw(self, a, k, n, sign):
        """a * exp(sign * 2 pi i k / n), folding the trivial angles."""
        k %= n
        if k == 0:
            return a
        if 4 * k == n:
            return self.mul_i(a) if sign > 0 else self.mul_mi(a)
        if 2 * k == n:
            return (self.neg(a[0]), self.neg(a[1]))
        if 4 * k == 3 * n:
            return self.mul_mi(a) if sign > 0 else self.mul_i(a)
        ang = 2.0 * math.pi * k / n
        cd, sd = math.cos(ang), sign * math.sin(ang)
        # Tangent form: (ar + i ai)(c + i s) = c [(ar - t ai) + i (ai + t ar)]
        # with t = s / c (or s [(t ar - ai) + i (ar + t ai)], t = c / s, when
        # |s| > |c|): one multiply-add per component, and the common factor
        # a multiply that the emitter folds into the adds consuming it.
        if abs(cd) >= abs(sd):
            t, m = float(np.float32(sd / cd)), float(np.float32(cd))
            re = self.mulc(self.fmac_common(a[1], -t, a[0]), m)
            im = self.mulc(self.fmac_common(a[0], t, a[1]), m)
        else:
            t, m = float(np.float32(cd / sd)), float(np.float32(sd))
            re = self.mulc(self.fmac_common(a[0], t, self.neg(a[1])), m)
            im = self.mulc(self.fmac_common(a[1], t, a[0]), m)
        return (re, im)


def rdft(g: Graph, x, top=True):
    """Real DFT of x (list of R, len n): returns X_k as (re, im) for
    k = 0..n/2 (X_0 and X_{n/2} real).  Below the top level the outputs may
    carry a constant factor (a multiply node) that the parent folds into
    its own operations."""
    n = len(x)
    if n == 1:
        return [(x[0], ZERO)]
    if n == 2:
        return [(g.add(x[0], x[1]), ZERO), (g.sub(x[0], x[1]), ZERO)]
    e = rdft(g, x[0::2], False)  # n/2: k = 0..n/4
    u = rdft(g, x[1::4], False)  # n/4: k = 0..n/8
    v = rdft(g, x[3::4], False)
    cadd = g.cadd if top else g.cadd_common
    csub = g.csub if top else g.csub_common

    def full(h, m, k):  # value at k of a Hermitian spectrum of length m
        k %= m
        return h[k] if k <= m // 2 else Graph.conj(h[m - k])

    out = [None] * (n // 2 + 1)
    q = n // 4
    # A_k = W^k U_k, B_k = W^3k V_k for k <= n/8; the rest by symmetry:
    # A_{q-k} = -i conj(A_k), B_{q-k} = +i conj(B_k).
    a = {}
    b = {}
    for k in range(0, n // 8 + 1):
        a[k] = g.ctw(full(u, q, k), k, n, -1)
        b[k] = g.ctw(full(v, q, k), 3 * k, n, -1)
    for k in range(n // 8 + 1, q):
        a[k] = Graph.mul_mi(Graph.conj(a[q - k]))
        b[k] = Graph.mul_i(Graph.conj(b[q - k]))
    for k in range(0, q):
        s = (g.add_common(a[k][0], b[k][0]), g.add_common(a[k][1], b[k][1]))
        dd = (g.add_common(a[k][0], b[k][0], -1), g.add_common(a[k][1], b[k][1], -1))
        out[k] = cadd(full(e, n // 2, k), s)
        out[k + q] = cadd(full(e, n // 2, k + q), Graph.mul_mi(dd))
    s0 = g.cadd_common(a[0], b[0])
    out[n // 2] = csub(full(e, n // 2, 0), s0)
    return out


def irdft(g: Graph, xs):
    """Inverse of rdft's spectrum: xs = X_k for k = 0..n/2 (Hermitian);
    returns x_m = sum_{k<n} X_k exp(+2 pi i k m / n), m = 0..n-1."""
    n = 2 * (len(xs) - 1)
    if n == 1 or len(xs) == 1:
        return [xs[0][0]]
    if n == 2:
        return [g.add_common(xs[0][0], xs[1][0]), g.add_common(xs[0][0], xs[1][0], -1)]

    def full(k):
        k %= n
        return xs[k] if k <= n // 2 else Graph.conj(xs[n - k])

    q = n // 4
    ep = [g.cadd_common(full(k), full(k + n // 2)) for k in range(0, q + 1)]
    up, vp = [], []
    for k in range(0, n // 8 + 1):
        d1 = g.csub_common(full(k), full(k + n // 2))
        d2 = g.csub_common(full(k + q), full(k + 3 * q))
        up.append(g.ctw(g.cadd_common(d1, Graph.mul_i(d2)), k, n, +1))
        vp.append(g.ctw(g.csub_common(d1, Graph.mul_i(d2)), 3 * k, n, +1))
    xe = irdft(g, ep)
    xu = irdft(g, up)
    xv = irdft(g, vp)
    x = [None] * n
    x[0::2] = xe
    x[1::4] = xu
    x[3::4] = xv
    return x


R2 = float(np.float32(math.sqrt(2.0)))
R2I = float(np.float32(1.0 / math.sqrt(2.0)))


def build_forward(n):
    g = Graph()
    x = [g.inp(f"x[{i}]") for i in range(n)]
    xs = rdft(g, x)
    outs = [g.mulc(xs[0][0], R2I), g.mulc(xs[n // 2][0], R2I)]
    for k in range(1, n // 2):
        outs += [xs[k][0], xs[k][1]]
    return g, outs


def transpose(g: Graph, outs, n, in_name, out_name):
    """The adjoint of the linear map x -> outs (inputs named in_name[i]):
    a graph from inputs out_name[j] to n outputs, each original edge
    reversed with its coefficient (a fan-out becomes a sum).  Same number
    of operations as the original, give or take its input/output counts."""
    live = live_nodes(g, outs)
    cons = {i: [] for i in live}  # node -> [(consumer, coefficient)]
    for i in sorted(live):
        op, args = g.nodes[i]
        if op == "add":
            cons[args[0]].append((i, 1.0))
            cons[args[1]].append((i, 1.0))
        elif op == "sub":
            cons[args[0]].append((i, 1.0))
            cons[args[1]].append((i, -1.0))
        elif op == "mul":
            cons[args[0]].append((i, args[1]))
        elif op == "fma":
            cons[args[0]].append((i, args[1]))
            cons[args[2]].append((i, 1.0))
    gt = Graph()
    seeds = {i: [] for i in live}
    for j, o in enumerate(outs):
        if o.node is not None:
            seeds[o.node].append(gt.mulc(gt.inp(f"{out_name}[{j}]"), float(o.sign)))
    tval = {}
    for i in sorted(live, reverse=True):  # every consumer has a larger index
        terms = [(t, 1.0) for t in seeds[i]] + [(tval[c], w) for c, w in cons[i]]

        def scaled(tw):  # a term that would start the sum with a factor
            t, w = tw
            return abs(w) != 1.0 or gt.split_mul(t)[1] is not None

        terms.sort(key=scaled)  # an unscaled term first: no factor to carry
        acc = ZERO
        for t, w in terms:
            acc = gt.fmac_common(t, w, acc) if acc.node is not None else gt.mulc(t, w)
        tval[i] = acc
    res = []
    for k in range(n):
        key = ("in", (f"{in_name}[{k}]",))
        node = g.memo.get(key)
        res.append(tval.get(node, ZERO) if node is not None else ZERO)
    return gt, res


def build_inverse(n):
    """The adjoint of build_forward: x = A^T y (half the unnormalized inverse
    real DFT of the packed spectrum y)."""
    g, outs = build_forward(n)
    return transpose(g, outs, n, "x", "y")


def evaluate(g: Graph, outs, inputs: dict):
    vals = {}
    for i, (op, args) in enumerate(g.nodes):
        if op == "in":
            vals[i] = inputs[args[0]]
        elif op == "add":
            vals[i] = vals[args[0]] + vals[args[1]]
        elif op == "sub":
            vals[i] = vals[args[0]] - vals[args[1]]
        elif op == "mul":
            vals[i] = vals[args[0]] * args[1]
        elif op == "fma":
            vals[i] = vals[args[0]] * args[1] + vals[args[2]]
    res = []
    for o in outs:
        res.append(0.0 if o.node is None else o.sign * vals[o.node])
    return np.array(res)


def live_nodes(g: Graph, outs):
    live = set()
    stack = [o.node for o in outs if o.node is not None]
    while stack:
        i = stack.pop()
        if i in live:
            continue
        live.add(i)
        op, args = g.nodes[i]
        if op in ("add", "sub"):
            stack += [args[0], args[1]]
        elif op == "mul":
            stack.append(args[0])
        elif op == "fma":
            stack += [args[0], args[2]]
    return live


def check(n):
    rng = np.random.default_rng(n)
    xv = rng.standard_normal((4, n))
    g, outs = build_forward(n)
    X = np.fft.rfft(xv, axis=1)
    for r in range(4):
        got = evaluate(g, outs, {f"x[{i}]": xv[r, i] for i in range(n)})
        ref = np.empty(n)
        ref[0] = X[r, 0].real / math.sqrt(2)
        ref[1] = X[r, n // 2].real / math.sqrt(2)
        ref[2::2] = X[r, 1:n // 2].real
        ref[3::2] = X[r, 1:n // 2].imag
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err < 1e-6, (n, "forward", err)
    gi, outi = build_inverse(n)
    for r in range(4):
        yv = rng.standard_normal(n)
        got = evaluate(gi, outi, {f"y[{i}]": yv[i] for i in range(n)})
        Xs = np.zeros(n // 2 + 1, complex)
        Xs[0] = yv[0] * math.sqrt(2)
        Xs[n // 2] = yv[1] * math.sqrt(2)
        Xs[1:n // 2] = yv[2::2][: n // 2 - 1] + 1j * yv[3::2][: n // 2 - 1]
        ref = np.fft.irfft(Xs, n) * (n / 2)
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err < 1e-6, (n, "inverse", err)


def fmt(c: float) -> str:
    return f"{np.float32(c).item():.9e}f"


def use_counts(g: Graph, outs, live):
    uses = {i: 0 for i in live}
    for i in live:
        op, args = g.nodes[i]
        if op in ("add", "sub"):
            uses[args[0]] += 1
            uses[args[1]] += 1
        elif op == "mul":
            uses[args[0]] += 1
        elif op == "fma":
            uses[args[0]] += 1
            uses[args[2]] += 1
    for o in outs:
        if o.node is not None:
            uses[o.node] += 1
    return uses


def emit_x2(name, g: Graph, outs, in_arr, out_arr, n):
    """Two-lane version of `emit`: every value is an f2 (two independent
    transforms in lock step, constants broadcast to both lanes), built only
    from add/sub/mul/fma.rn.f32x2, which take no negated operands.  Each
    emitted value therefore carries a polarity p (the register holds p times
    the true value), chosen per operation so that one instruction suffices;
    the polarity of every output is returned for the caller to absorb.
    Returns (code, op count, output polarities, op list for `run_x2`)."""
    live = live_nodes(g, outs)
    # A multiply by a constant whose every consumer is an add/sub disappears:
    # each consumer becomes one multiply-add (same cost as the add).
    users = {i: [] for i in live}
    for i in sorted(live):
        op, args = g.nodes[i]
        if op in ("add", "sub"):
            users[args[0]].append(i)
            users[args[1]].append(i)
        elif op == "mul":
            users[args[0]].append(i)
        elif op == "fma":
            users[args[0]].append(i)
            users[args[2]].append(i)
    out_nodes = {o.node for o in outs if o.node is not None}
    fused = {}
    absorbed = set()
    for m in sorted(live):
        if g.nodes[m][0] != "mul" or m in out_nodes or not users[m]:
            continue
        us = users[m]
        if len(set(us)) != len(us) or any(
                g.nodes[i][0] not in ("add", "sub") or i in fused for i in us):
            continue
        for i in us:
            op, args = g.nodes[i]
            pos = 1 if args[1] == m else 0
            other = args[1 - pos]
            if op == "add":
                fused[i] = (m, +1, other, +1)
            elif pos == 1:
                fused[i] = (m, -1, other, +1)
            else:
                fused[i] = (m, +1, other, -1)
        absorbed.add(m)
    pol = {}
    prog = []  # (dst, op, a, b, const): op in add/sub/mul/fma; fma = a*const + b
    lines = [f"__device__ __forceinline__ void {name}(const f2 (&{in_arr})[{n}], "
             f"f2 (&{out_arr})[{n}]) {{"]

    def ref(i):
        op, args = g.nodes[i]
        return args[0] if op == "in" else f"t{i}"

    def lin(i, a, ca, b, cb):
        """value = ca*a + cb*b (ca a constant, cb = +-1) as one fma."""
        cb_eff = cb * pol[b]
        c_eff = ca * pol[a]
        if cb_eff > 0:
            return ("fma", a, b, c_eff, +1)
        return ("fma", a, b, -c_eff, -1)

    counts = {"add": 0, "sub": 0, "mul": 0, "fma": 0}
    for i, (op, args) in enumerate(g.nodes):
        if i not in live or i in absorbed:
            continue
        if op == "in":
            pol[i] = +1
            continue
        if i in fused:
            m, msign, other, osign = fused[i]
            src, c = g.nodes[m][1]
            kind, a, b, cc, p = lin(i, src, msign * c, other, osign)
        elif op == "fma":
            kind, a, b, cc, p = lin(i, args[0], args[1], args[2], +1)
        elif op == "mul":
            kind, a, b, cc, p = "mul", args[0], None, args[1] * pol[args[0]], +1
        else:
            x, y = args
            sy = +1 if op == "add" else -1
            px, py = pol[x], pol[y] * sy  # value = px*X' + py*Y'
            if px > 0 and py > 0:
                kind, a, b, p = "add", x, y, +1
            elif px > 0:
                kind, a, b, p = "sub", x, y, +1
            elif py > 0:
                kind, a, b, p = "sub", y, x, +1
            else:
                kind, a, b, p = "add", x, y, -1
            cc = None
        pol[i] = p
        prog.append((i, kind, a, b, cc))
        counts[kind] += 1
        if kind == "add":
            e = f"add2({ref(a)}, {ref(b)})"
        elif kind == "sub":
            e = f"sub2({ref(a)}, {ref(b)})"
        elif kind == "mul":
            e = f"mul2({ref(a)}, mk2({fmt(cc)}, {fmt(cc)}))"
        else:
            e = f"fma2({ref(a)}, mk2({fmt(cc)}, {fmt(cc)}), {ref(b)})"
        lines.append(f"  const f2 t{i} = {e};")
    opol = []
    for j, o in enumerate(outs):
        if o.node is None:
            lines.append(f"  {out_arr}[{j}] = mk2(0.0f, 0.0f);")
            opol.append(+1)
        else:
            lines.append(f"  {out_arr}[{j}] = {ref(o.node)};")
            opol.append(o.sign * pol[o.node])
    lines.append("}")
    total = sum(counts.values())
    head = (f"// {name}: {counts['add'] + counts['sub']} add/sub, {counts['mul']} mul, "
            f"{counts['fma']} fma ({total} f32x2 instructions)")
    outs_nodes = [o.node for o in outs]
    return head + "\n" + "\n".join(lines) + "\n", total, opol, (prog, outs_nodes)


def run_x2(g: Graph, prog, outs_nodes, inputs: dict):
    """Interpret an emit_x2 op list (one lane) on numbers: returns the
    stored (polarity-scaled) outputs."""
    vals = {}
    for i, (op, args) in enumerate(g.nodes):
        if op == "in":
            vals[i] = inputs[args[0]]
    for dst, kind, a, b, cc in prog:
        if kind == "add":
            vals[dst] = vals[a] + vals[b]
        elif kind == "sub":
            vals[dst] = vals[a] - vals[b]
        elif kind == "mul":
            vals[dst] = vals[a] * cc
        else:
            vals[dst] = vals[a] * cc + vals[b]
    return np.array([0.0 if nd is None else vals[nd] for nd in outs_nodes])


def check_x2(n, g, outs, prog_outs, opol, forward):
    """The emitted two-lane program, polarities applied, equals the graph."""
    rng = np.random.default_rng(100 + n)
    prog, onodes = prog_outs
    name = "x" if forward else "y"
    for _ in range(4):
        xv = rng.standard_normal(n)
        inputs = {f"{name}[{i}]": xv[i] for i in range(n)}
        ref = evaluate(g, outs, inputs)
        got = run_x2(g, prog, onodes, inputs) * np.array(opol)
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err < 1e-12, (n, forward, err)


def pol_mask(opol):
    return sum(1 << j for j, p in enumerate(opol) if p < 0)


def main(path=None):
    here = os.path.dirname(os.path.abspath(__file__))
    path = path or os.path.join(here, "kvq_rfft.cuh")
    parts = [
        "// kvq_rfft.cuh -- GENERATED by gen_rfft.py; do not edit by hand.\n",
        "// Two-lane real-input split-radix FFT codelets (see gen_rfft.py).\n",
        "#pragma once\n\nnamespace kvq {\n\n",
        "template <int N> struct RFFT2;\n\n",
    ]
    for n in (32, 64):
        check(n)
        gf, of = build_forward(n)
        gi, oi = build_inverse(n)
        fwd, cf, pf, progf = emit_x2(f"rfft{n}x2_fwd", gf, of, "x", "y", n)
        inv, ci, pi, progi = emit_x2(f"rfft{n}x2_inv", gi, oi, "y", "x", n)
        check_x2(n, gf, of, progf, pf, True)
        check_x2(n, gi, oi, progi, pi, False)
        parts += [fwd, "\n", inv, "\n"]
        parts.append(
            f"// Two independent {n}-point transforms in the two lanes of each f2.\n"
            f"// Output j holds -1 times its true value where bit j of FWD_NEG / INV_NEG\n"
            f"// is set.\n"
            f"template <> struct RFFT2<{n}> {{\n"
            f"  static constexpr uint64_t FWD_NEG = 0x{pol_mask(pf):016x}ull;\n"
            f"  static constexpr uint64_t INV_NEG = 0x{pol_mask(pi):016x}ull;\n"
            f"  static __device__ __forceinline__ void fwd(const f2 (&x)[{n}], f2 (&y)[{n}]) "
            f"{{ rfft{n}x2_fwd(x, y); }}\n"
            f"  static __device__ __forceinline__ void inv(const f2 (&y)[{n}], f2 (&x)[{n}]) "
            f"{{ rfft{n}x2_inv(y, x); }}\n"
            f"}};\n\n")
        print(f"n={n} x2: forward {cf} f32x2 ops, inverse {ci} f32x2 ops", file=sys.stderr)
    parts.append("}  // namespace kvq\n")
    with open(path, "w") as f:
        f.write("".join(parts))
    return path


if __name__ == "__main__":
    main()
