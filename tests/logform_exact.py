"""DeltaLog's deferred-materialization scheme in exact rational arithmetic.

Test-only restatement of the method ("DeltaLog: Deferred Materialization of
Recurrent States for Linear Attention Decoding", Abstract): the state is a
dense base plus a bounded log of compact rank-1 factors; each decode step
reads base + log, appends one factor instead of writing the full state, and a
periodic merge folds the log back into the base.  The model must observe the
same dense state as eager decoding.

It is written independently of both the fp64 oracle (an eager recurrence)
and the CUDA kernels (fp32, log-space decay): here everything is a
``fractions.Fraction`` and the cumulative decay is kept as an exact product
Gamma, so ratios Gamma_t / Gamma_i are exact.  Comparing this with the
oracle on tiny inputs pins both: the algebra of the log form, and the
oracle's eager arithmetic.

Orientation: every state is d_v x d_k (row = value index, column = key
channel); for RWKV6 that is the transpose of its recurrence's d_k x d_v
matrix.
"""

from __future__ import annotations

from fractions import Fraction
from typing import List, Optional, Sequence

Vec = List[Fraction]
Mat = List[List[Fraction]]


def _dot(a: Sequence[Fraction], b: Sequence[Fraction]) -> Fraction:
    return sum((x * y for x, y in zip(a, b)), Fraction(0))


class ExactDeltaLog:
    """One head of DeltaLog, exact.  ``variant`` in {"gdn", "kda", "rwkv6",
    "gdn2"}."""

    def __init__(self, variant: str, S0: Mat, L: int, fill0: int = 0,
                 bonus: Optional[Vec] = None):
        self.variant = variant
        self.dv = len(S0)
        self.dk = len(S0[0])
        self.L = L
        self.base: Mat = [[Fraction(x) for x in row] for row in S0]
        self.bonus = None if bonus is None else [Fraction(x) for x in bonus]
        one = self._unit_decay()
        # fill offsets: entries that change nothing (u = 0, k = 0, Gamma = 1)
        self.log = [([Fraction(0)] * self.dv, [Fraction(0)] * self.dk, one)
                    for _ in range(fill0)]

    # ---- decay bookkeeping: scalar for GDN, per key channel otherwise
    def _unit_decay(self):
        return Fraction(1) if self.variant == "gdn" else [Fraction(1)] * self.dk

    def _last_decay(self):
        return self.log[-1][2] if self.log else self._unit_decay()

    def _times(self, gamma, decay):
        if self.variant == "gdn":
            return gamma * Fraction(decay)
        return [g * Fraction(a) for g, a in zip(gamma, decay)]

    def _ratio_dot(self, k_i, x, gamma_t, gamma_i) -> Fraction:
        """sum_c k_i[c] x[c] Gamma_t[c] / Gamma_i[c] (scalar Gamma for GDN)."""
        if self.variant == "gdn":
            return (gamma_t / gamma_i) * _dot(k_i, x)
        return sum((k_i[c] * x[c] * gamma_t[c] / gamma_i[c] for c in range(self.dk)),
                   Fraction(0))

    def _base_times(self, x, gamma) -> Vec:
        """S_b (Gamma o x) -- Gamma scalar or per key channel."""
        if self.variant == "gdn":
            xs = [gamma * xc for xc in x]
        else:
            xs = [g * xc for g, xc in zip(gamma, x)]
        return [_dot(row, xs) for row in self.base]

    # ---- the decode step: reads base + log, appends one factor
    def step(self, q, k, v, decay, beta=None, wgate=None) -> Vec:
        """GDN-2: ``beta`` is the erase gate b (per key channel) and
        ``wgate`` the write gate w (per value row): the read key is b o k and
        the written value w o v, u_t = w o v - S'(b o k)."""
        if len(self.log) >= self.L:
            raise RuntimeError("log full: merge first")
        q = [Fraction(x) for x in q]
        k = [Fraction(x) for x in k]
        v = [Fraction(x) for x in v]
        gprev = self._last_decay()
        gt = self._times(gprev, decay)
        if self.variant == "rwkv6":
            # readout of S_{t-1} (decay Gamma_prev), then the bonus term
            o = self._base_times(q, gprev)
            for (u_i, k_i, g_i) in self.log:
                coef = self._ratio_dot(k_i, q, gprev, g_i)
                o = [oj + coef * uj for oj, uj in zip(o, u_i)]
            bonus = sum((q[c] * self.bonus[c] * k[c] for c in range(self.dk)), Fraction(0))
            o = [oj + bonus * vj for oj, vj in zip(o, v)]
            self.log.append((v, k, gt))
            return o
        if self.variant == "gdn2":
            kread = [Fraction(bc) * kc for bc, kc in zip(beta, k)]
        else:
            beta = Fraction(beta)
            kread = k
        a = self._base_times(kread, gt)
        b = self._base_times(q, gt)
        for (u_i, k_i, g_i) in self.log:
            ck = self._ratio_dot(k_i, kread, gt, g_i)
            cq = self._ratio_dot(k_i, q, gt, g_i)
            a = [aj + ck * uj for aj, uj in zip(a, u_i)]
            b = [bj + cq * uj for bj, uj in zip(b, u_i)]
        if self.variant == "gdn2":
            u_t = [Fraction(wj) * vj - aj for wj, vj, aj in zip(wgate, v, a)]
        else:
            u_t = [beta * (vj - aj) for vj, aj in zip(v, a)]
        kq = _dot(k, q)
        o = [bj + kq * uj for bj, uj in zip(b, u_t)]
        self.log.append((u_t, k, gt))
        return o

    # ---- materialize / merge
    def dense(self) -> Mat:
        """S_t = S_b Diag(Gamma) + sum_i u_i (k_i o Gamma / Gamma_i)^T."""
        if not self.log:
            return [row[:] for row in self.base]
        gl = self._last_decay()
        if self.variant == "gdn":
            col = [gl] * self.dk
        else:
            col = list(gl)
        S = [[self.base[j][c] * col[c] for c in range(self.dk)] for j in range(self.dv)]
        for (u_i, k_i, g_i) in self.log:
            for c in range(self.dk):
                r = (gl / g_i) if self.variant == "gdn" else (gl[c] / g_i[c])
                kc = k_i[c] * r
                if kc == 0:
                    continue
                for j in range(self.dv):
                    S[j][c] += u_i[j] * kc
        return S

    def merge(self) -> None:
        self.base = self.dense()
        self.log = []

    @property
    def fill(self) -> int:
        return len(self.log)
