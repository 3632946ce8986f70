"""GPU-vs-oracle parity harness (test infrastructure).

Runs the library's decode paths through the C ABI on the seeded inputs of a
workload, and the fp64 oracle on the same inputs for a sample of heads (every
head is an independent recurrence, so a sample checks the full launch
exactly), then reports the relative errors north of which a test fails:

  state : max |S_gpu - S_ref| / max |S_ref| over the checked heads, taken
          at every snapshot step (every ``snap_every`` steps and at T);
  output: max over steps t of max |o_gpu - o_ref| / max |o_ref| (over the
          checked heads and value rows).

Several "arms" run in one pass over the inputs so the draws are made once:
  "log"    DeltaLog step + dl_merge(DL_MERGE_FULL) after every step
  "fused"  DeltaLog step with the merge fused into the step kernel
  "eager"  the dense eager step kernel
"""

from __future__ import annotations

import dataclasses
import types
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle
from linear_attention_recurrent_deltalog_b200 import deltalog as dlb
from linear_attention_recurrent_deltalog_b200 import workloads as wl

STATE_TOL = 1e-4
OUT_TOL = 1e-3


def host_to_device(x: np.ndarray, dev) -> torch.Tensor:
    """numpy array as the kernel reads it (uint16 -> bf16 bits, else fp32)."""
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)


def step_to_device(s: wl.StepInputs, dev):
    q = host_to_device(s.device_array("q"), dev).reshape(-1)
    k = host_to_device(s.device_array("k"), dev).reshape(-1)
    v = host_to_device(s.device_array("v"), dev).reshape(-1)
    dec = host_to_device(s.decay, dev).reshape(-1)
    beta = None if s.beta is None else host_to_device(s.beta, dev).reshape(-1)
    return q, k, v, dec, beta


def step_bonus(s: wl.StepInputs, dev, fixed=None):
    """The step's `bonus` argument: GDN-2's write gate for this step, else the
    fixed RWKV6 bonus (or None)."""
    if s.wgate is not None:
        return host_to_device(s.wgate, dev).reshape(-1)
    return fixed


@dataclasses.dataclass
class ArmResult:
    state_err: float
    out_err: float
    outputs: List[np.ndarray]
    states: Dict[int, np.ndarray]


_S0_CACHE: Dict[tuple, np.ndarray] = {}


def cached_initial_state(w: wl.Workload) -> np.ndarray:
    """wl.initial_state(w), memoised: it does not depend on L, and the 1 GiB
    draw of the serving batch takes several seconds."""
    key = (w.seed, w.B, w.H, w.d_v, w.d_k, w.s0_std)
    if key not in _S0_CACHE:
        if len(_S0_CACHE) > 2:
            _S0_CACHE.clear()
        _S0_CACHE[key] = wl.initial_state(w)
    return _S0_CACHE[key]


def _rel(a: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(a - ref))) / (den if den > 0 else 1.0)


def run_parity(w: wl.Workload, T: Optional[int] = None, heads: Optional[Sequence[int]] = None,
               arms=("log", "fused", "eager"), snap_every: int = 64, L: Optional[int] = None,
               merge_all_at: Sequence[int] = (), workers: Optional[int] = None,
               split: int = 0, device="cuda",
               edit=None) -> Dict[str, ArmResult]:
    """Runs the given arms and the oracle; returns per-arm errors.  ``edit``
    (optional) maps each drawn StepInputs to the one both sides receive."""
    if L is not None:
        w = w.replace(L=L)
    T = w.T if T is None else T
    BH, dk, dv = w.heads, w.d_k, w.d_v
    heads = np.arange(BH) if heads is None else np.asarray(heads, dtype=np.int64)
    heads_t = torch.from_numpy(heads).to(device)
    S0 = cached_initial_state(w)
    fill0 = wl.fill_offsets(w)
    bonus = wl.rwkv6_bonus(w) if w.variant == wl.RWKV6 else None
    bonus_d = None if bonus is None else torch.from_numpy(bonus).to(device).reshape(-1)
    S0_d = torch.from_numpy(S0).to(device).reshape(-1)
    snaps = sorted(set([t for t in range(snap_every, T + 1, snap_every)] + [T]))

    states = {}
    dense = {}
    for arm in arms:
        if arm == "eager":
            dense[arm] = S0_d.clone()
        else:
            cfg = dlb.Config(w.variant, w.B, w.H, dk, dv, w.L, w.in_dtype,
                             fused_merge=(arm == "fused"), step_split=split,
                             kla_eps=w.kla_eps)
            st = dlb.DeltaLogState(cfg, device=device)
            st.reset(S0_d, fill0.tolist())
            states[arm] = st
    cfg_e = dlb.Config(w.variant, w.B, w.H, dk, dv, w.L, w.in_dtype, kla_eps=w.kla_eps)
    out = {arm: [] for arm in arms}
    snap_gpu = {arm: {} for arm in arms}
    recs = []
    o = torch.empty(BH * dv, dtype=torch.float32, device=device)
    S_out = torch.empty(BH * dv * dk, dtype=torch.float32, device=device)
    for s in wl.StepStream(w, T, workers=workers):
        if edit is not None:
            s = edit(s)
        q, k, v, dec, beta = step_to_device(s, device)
        bon_s = step_bonus(s, device, bonus_d)
        n = s.t + 1
        for arm in arms:
            if arm == "eager":
                dlb.dl_eager_step(cfg_e, dense[arm], q, k, v, dec, beta, bon_s, o)
            else:
                st = states[arm]
                st.step(q, k, v, dec, beta, bon_s, o)
                if arm == "log":
                    st.merge(dlb.DL_MERGE_FULL)
                if n in merge_all_at:
                    st.merge(dlb.DL_MERGE_ALL)
            out[arm].append(o.view(BH, dv).index_select(0, heads_t).cpu().numpy().astype(np.float64))
            if n in snaps:
                if arm == "eager":
                    S = dense[arm]
                else:
                    states[arm].materialize(S_out)
                    S = S_out
                snap_gpu[arm][n] = (S.view(BH, dv, dk).index_select(0, heads_t).cpu().numpy()
                                    .astype(np.float64))
        flat = lambda x: None if x is None else x.reshape((BH,) + x.shape[2:])[heads][:, None]
        recs.append(types.SimpleNamespace(q=flat(s.q), k=flat(s.k), v=flat(s.v),
                                          decay=flat(s.decay), beta=flat(s.beta),
                                          wgate=flat(s.wgate)))
    torch.cuda.synchronize()
    for arm, st in states.items():
        code, head = st.device_error()
        assert code == 0, f"device error {code} at head {head} ({arm})"
        st.close()

    S0h = S0.reshape(BH, dv, dk)[heads].astype(np.float64)
    if w.variant == wl.RWKV6:
        S0h = S0h.transpose(0, 2, 1)
    bon = None if bonus is None else bonus[heads % w.H]
    ref = oracle.run_eager(w.variant, S0h, recs, bonus=bon, snapshot_at=snaps, kla_eps=w.kla_eps)
    result = {}
    for arm in arms:
        out_err = max(_rel(a, r) for a, r in zip(out[arm], ref.outputs))
        st_err = 0.0
        for n in snaps:
            Sr = ref.states[n]
            if w.variant == wl.RWKV6:
                Sr = Sr.transpose(0, 2, 1)
            st_err = max(st_err, _rel(snap_gpu[arm][n], Sr))
        result[arm] = ArmResult(st_err, out_err, out[arm], snap_gpu[arm])
    return result


def heads_covering_phases(w: wl.Workload, n: int, L: Optional[int] = None) -> np.ndarray:
    """A seeded head sample that contains every fill offset present."""
    if L is not None:
        w = w.replace(L=L)
    fill = wl.fill_offsets(w)
    picked = []
    for f in sorted(set(fill.tolist())):
        b = int(np.nonzero(fill == f)[0][0])
        picked.append(b * w.H + (f % w.H))
    rest = wl.sample_heads(w, n)
    allh = np.unique(np.concatenate([np.array(picked, dtype=np.int64), rest]))
    return allh


# ------------------------------------------------------------- int8 base

@dataclasses.dataclass
class Q8Result:
    reset_exact: bool        # Q(S0) codes and scales bit-identical to the oracle's
    out_err: float           # as in run_parity, against the windowed oracle
    state_err: float         # materialized state against the windowed oracle
    code_excess: float       # max over requantized elements of
                             #   |code_gpu - x inv| - 0.5 - delta  (<= 0 passes)
    scale_excess: float      # max of |scale_gpu - scale_ref| - allowed  (<= 0 passes)
    mismatch_frac: float     # fraction of requantized codes that differ
    windows: int             # window ends checked


def _lib_rows(S, rec):
    return np.swapaxes(S, -1, -2) if rec else S


def run_parity_q8(w: wl.Workload, T: Optional[int] = None, heads: Optional[Sequence[int]] = None,
                  fused: bool = True, split: int = 0, merge_all_at: Sequence[int] = (),
                  resync: bool = True, snap_every: int = 8, workers: Optional[int] = 0,
                  device="cuda", edit=None) -> Q8Result:
    """The int8-base path against the windowed oracle (oracle.run_windowed's
    definition, stepped here one step at a time for the sampled heads).

    At every window end the GPU's new codes must be a correct rounding of
    the oracle's pre-quantization value x: |code - x inv| <= 0.5 + delta with
    delta = 2 eps inv, eps = STATE_TOL * max|x| over the head (the GPU's x
    and amax may differ from the oracle's by the state tolerance).  With
    ``resync`` the oracle's codes and scales are then written into the GPU
    base for those heads, so every window starts from identical values and
    outputs and states are held to the fp32 tolerances.  ``edit`` as in
    run_parity."""
    T = w.T if T is None else T
    BH, dk, dv, H, L = w.heads, w.d_k, w.d_v, w.H, w.L
    rec = w.variant == wl.RWKV6
    heads = np.arange(BH) if heads is None else np.asarray(heads, dtype=np.int64)
    heads_t = torch.from_numpy(heads).to(device)
    S0 = cached_initial_state(w)
    fill0 = wl.fill_offsets(w)
    bonus = wl.rwkv6_bonus(w) if rec else None
    bonus_d = None if bonus is None else torch.from_numpy(bonus).to(device).reshape(-1)
    bon = None if bonus is None else bonus[heads % H]
    cfg = dlb.Config(w.variant, w.B, H, dk, dv, L, w.in_dtype, fused_merge=fused, step_split=split,
                     kla_eps=w.kla_eps, base="q8")
    st = dlb.DeltaLogState(cfg, device=device)
    st.reset(torch.from_numpy(S0).to(device).reshape(-1), fill0.tolist())
    S0h = S0.reshape(BH, dv, dk)[heads]
    c0, s0 = oracle.quantize_rows(S0h)
    g_codes = st.base_codes(heads_t).cpu().numpy()
    g_scales = st.base_scales().index_select(0, heads_t).cpu().numpy()
    reset_exact = bool(np.array_equal(g_codes, c0) and np.array_equal(g_scales, s0))
    S = _lib_rows(oracle.dequantize_rows(c0, s0), rec).copy()      # recurrence orientation
    fill = fill0[heads // H].astype(np.int64)
    o = torch.empty(BH * dv, dtype=torch.float32, device=device)
    S_out = torch.empty(BH * dv * dk, dtype=torch.float32, device=device)
    out_err = state_err = 0.0
    code_excess = scale_excess = -np.inf
    mismatches = total = windows = 0
    forced = set(int(x) for x in merge_all_at)
    for s in wl.StepStream(w, T, workers=workers):
        if edit is not None:
            s = edit(s)
        q, k, v, dec, beta = step_to_device(s, device)
        n = s.t + 1
        st.step(q, k, v, dec, beta, step_bonus(s, device, bonus_d), o)
        if not fused:
            st.merge(dlb.DL_MERGE_FULL)
        if n in forced:
            st.merge(dlb.DL_MERGE_ALL)
        o_gpu = o.view(BH, dv).index_select(0, heads_t).cpu().numpy().astype(np.float64)
        flat = lambda x: None if x is None else x.reshape((BH,) + x.shape[2:])[heads][:, None]
        step = types.SimpleNamespace(q=flat(s.q), k=flat(s.k), v=flat(s.v), decay=flat(s.decay),
                                     beta=flat(s.beta), wgate=flat(s.wgate))
        res = oracle.run_eager(w.variant, S, [step], bonus=bon, kla_eps=w.kla_eps)
        S = res.S
        out_err = max(out_err, _rel(o_gpu, res.outputs[0]))
        fill += 1
        ended = (fill > 0) if n in forced else (fill == L)
        idx = np.nonzero(ended)[0]
        if idx.size:
            pre = _lib_rows(S[idx], rec)
            codes, scales = oracle.quantize_rows(pre)
            inv = oracle.row_inverse(pre).astype(np.float64)
            gidx = torch.from_numpy(heads[idx]).to(device)
            gc = st.base_codes(gidx).cpu().numpy().astype(np.float64)
            gs = st.base_scales().index_select(0, gidx).cpu().numpy().astype(np.float64)
            eps = STATE_TOL * np.max(np.abs(pre), axis=(1, 2), keepdims=True)
            delta = 2.0 * eps * inv[..., None] + 1e-6
            dev_c = np.abs(gc - pre * inv[..., None]) - 0.5 - delta
            code_excess = max(code_excess, float(np.max(dev_c)))
            dev_s = np.abs(gs - scales) - (eps[..., 0] / 127.0 * 1.0001 + 1e-30)
            scale_excess = max(scale_excess, float(np.max(dev_s)))
            mismatches += int(np.count_nonzero(gc != codes))
            total += codes.size
            windows += idx.size
            if resync:
                st.set_base_codes(gidx, torch.from_numpy(codes))
                st.base_scales().index_copy_(0, gidx, torch.from_numpy(scales).to(device))
            S[idx] = _lib_rows(oracle.dequantize_rows(codes, scales), rec)
            fill[idx] = 0
        if n % snap_every == 0 or n == T:
            st.materialize(S_out)
            Sg = S_out.view(BH, dv, dk).index_select(0, heads_t).cpu().numpy().astype(np.float64)
            state_err = max(state_err, _rel(Sg, _lib_rows(S, rec)))
    torch.cuda.synchronize()
    code, head = st.device_error()
    assert code == 0, f"device error {code} at head {head}"
    st.close()
    return Q8Result(reset_exact, out_err, state_err, code_excess, scale_excess,
                    mismatches / max(total, 1), windows)
