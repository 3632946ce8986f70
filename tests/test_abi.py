"""The C ABI library without a GPU (CPU only): it loads, exports every
declared symbol, sizes buffers, and rejects bad arguments on the host before
any CUDA call."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

from linear_attention_recurrent_deltalog_b200 import deltalog as dlb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "deltalog.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dl_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(dlb.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"missing export {n}"
    assert sorted(dlb.EXPORTED) == names


def test_status_strings():
    assert dlb.dl_status_string(0) == "ok"
    assert "merge" in dlb.dl_status_string(dlb.DL_ERR_LOG_FULL)
    assert dlb.dl_status_string(-99) == "unknown status"


def cfg(**kw):
    base = dict(variant="gdn", B=4, H=2, d_k=128, d_v=128, L=16, in_dtype="bf16")
    base.update(kw)
    return dlb.Config(**base)


def test_state_bytes_layout():
    c = cfg()
    nb, nl, nm = dlb.dl_state_bytes(c)
    BH = 8
    assert nb == BH * 128 * 128 * 4
    # u fp32 + k bf16 + scalar g, each array 256-B padded
    pad = lambda x: (x + 255) // 256 * 256
    assert nl == pad(BH * 16 * 128 * 4) + pad(BH * 16 * 128 * 2) + pad(BH * 16 * 4)
    # GDN's scalar log-decay stride is padded to a multiple of 4 entries
    _, nl5, _ = dlb.dl_state_bytes(cfg(L=5))
    assert nl5 == pad(BH * 5 * 128 * 4) + pad(BH * 5 * 128 * 2) + pad(BH * 8 * 4)
    assert nm == 2 * pad(BH * 4) + 256  # two fill arrays (step parity) + error word
    # KDA: vector log-decay; RWKV6: u stored in the input dtype
    _, nl_kda, _ = dlb.dl_state_bytes(cfg(variant="kda"))
    assert nl_kda == pad(BH * 16 * 128 * 4) + pad(BH * 16 * 128 * 2) + pad(BH * 16 * 128 * 4)
    _, nl_rw, _ = dlb.dl_state_bytes(cfg(variant="rwkv6", d_k=64, d_v=64, L=32))
    assert nl_rw == pad(BH * 32 * 64 * 2) + pad(BH * 32 * 64 * 2) + pad(BH * 32 * 64 * 4)
    # GDN-2 keeps KDA's log
    assert dlb.dl_state_bytes(cfg(variant="gdn2")) == dlb.dl_state_bytes(cfg(variant="kda"))
    # int8 base: codes, then the fp32 row scales at the next 256-B boundary;
    # the log and meta buffers do not change
    nbq, nlq, nmq = dlb.dl_state_bytes(cfg(base="q8"))
    assert nbq == pad(BH * 128 * 128) + pad(BH * 128 * 4)
    assert (nlq, nmq) == (nl, nm)
    nbq, _, _ = dlb.dl_state_bytes(cfg(base="q8", B=3, H=1, d_k=64, d_v=64))
    assert nbq == pad(3 * 64 * 64) + pad(3 * 64 * 4)


@pytest.mark.parametrize("bad,code", [
    (dict(variant="gdn", d_k=96), dlb.DL_ERR_UNSUPPORTED),
    (dict(L=0), dlb.DL_ERR_ARG),
    (dict(L=65), dlb.DL_ERR_ARG),
    (dict(B=0), dlb.DL_ERR_ARG),
    (dict(H=-1), dlb.DL_ERR_ARG),
    (dict(step_split=3), dlb.DL_ERR_ARG),
    (dict(step_split=4, d_v=64), dlb.DL_ERR_ARG),
    (dict(step_split=8), dlb.DL_ERR_ARG),
    # an int8 base needs work items of at least 64 rows
    (dict(step_split=4, base="q8"), dlb.DL_ERR_ARG),
    (dict(step_split=2, d_v=64, base="q8"), dlb.DL_ERR_ARG),
])
def test_state_bytes_rejects(bad, code):
    with pytest.raises(dlb.DeltaLogError) as e:
        dlb.dl_state_bytes(cfg(**bad))
    assert e.value.status == code


def test_bad_enums_rejected():
    c = cfg().c()
    c.variant = 7
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    c = cfg().c()
    c.in_dtype = 3
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    c = cfg().c()
    c.flags = 16
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    # bit 2 is reserved
    c = cfg().c()
    c.flags = 2
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    c = cfg(base="q8").c()
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_OK
    with pytest.raises(ValueError):
        cfg(base="q4").c()
    # the KLA step size applies to GDN and KDA, with a non-negative epsilon
    c = cfg(kla_eps=1e-6).c()
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_OK
    c = cfg(variant="rwkv6", d_k=64, d_v=64, kla_eps=1e-6).c()
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    c = cfg(kla_eps=-1.0).c()
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    # GDN-2: built for both bases; no KLA step size
    for base in ("f32", "q8"):
        c = cfg(variant="gdn2", base=base).c()
        assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_OK
    c = cfg(variant="gdn2", kla_eps=1e-6).c()
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG
    c = cfg().c()
    c.variant = 4
    assert dlb._lib.dl_state_bytes(ctypes.byref(c), None, None, None) == dlb.DL_ERR_ARG


def test_create_checks_pointers_without_touching_cuda():
    c = cfg()
    # fake device addresses: create only validates and stores them
    with pytest.raises(dlb.DeltaLogError) as e:
        dlb.dl_state_create(c, 0x1000, 0x2000, 0x3008)
    assert e.value.status == dlb.DL_ERR_ALIGN
    with pytest.raises(dlb.DeltaLogError) as e:
        dlb.dl_state_create(c, 0x1000, None, 0x3000)
    assert e.value.status == dlb.DL_ERR_ARG
    h = dlb.dl_state_create(c, 0x100000, 0x200000, 0x300000)
    try:
        assert dlb.dl_state_fill(h, c) == [0] * c.B
        # step argument checks happen before any launch
        st = dlb._lib.dl_decode_step
        assert st(h, None, 0x1000, 0x1000, 0x1000, 0x1000, None, 0x1000, None) == dlb.DL_ERR_ARG
        assert st(h, 0x1008, 0x1000, 0x1000, 0x1000, 0x1000, None, 0x1000, None) == dlb.DL_ERR_ALIGN
        # GDN needs beta
        assert st(h, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x1000, None) == dlb.DL_ERR_ARG
        assert dlb._lib.dl_merge(h, 5, None) == dlb.DL_ERR_ARG
        # nothing to merge: no launch, OK even without a GPU
        assert dlb._lib.dl_merge(h, dlb.DL_MERGE_FULL, None) == 0
        assert dlb._lib.dl_merge(h, dlb.DL_MERGE_ALL, None) == 0
        assert dlb._lib.dl_materialize(h, None, None) == dlb.DL_ERR_ARG
        assert dlb._lib.dl_materialize(h, 0x1004, None) == dlb.DL_ERR_ALIGN
        assert dlb._lib.dl_materialize(h, 0x100000, None) == dlb.DL_ERR_ARG  # aliases the base
        # reset rejects fill offsets outside [0, L)
        bad = (ctypes.c_int32 * c.B)(0, 16, 0, 0)
        assert dlb._lib.dl_state_reset(h, None, bad, None) == dlb.DL_ERR_ARG
    finally:
        dlb.dl_state_destroy(h)
    dlb.dl_state_destroy(None)


def test_rwkv6_needs_bonus():
    c = cfg(variant="rwkv6", d_k=64, d_v=64, L=32)
    h = dlb.dl_state_create(c, 0x100000, 0x200000, 0x300000)
    try:
        st = dlb._lib.dl_decode_step
        assert st(h, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x1000, None) == dlb.DL_ERR_ARG
    finally:
        dlb.dl_state_destroy(h)
    ec = cfg(variant="rwkv6", d_k=64, d_v=64).c()
    assert dlb._lib.dl_eager_step(ctypes.byref(ec), 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None,
                                  None, 0x1000, None) == dlb.DL_ERR_ARG


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="host without a GPU only")
def test_launch_failure_leaves_host_mirror_unchanged():
    # Without a device the launch fails with DL_ERR_CUDA; the fill mirror
    # must not advance.
    c = cfg()
    h = dlb.dl_state_create(c, 0x100000, 0x200000, 0x300000)
    try:
        rc = dlb._lib.dl_decode_step(h, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, 0x1000, None)
        assert rc == dlb.DL_ERR_CUDA
        assert dlb.dl_state_fill(h, c) == [0] * c.B
    finally:
        dlb.dl_state_destroy(h)


def test_binding_rejects_undersized_tensors():
    import torch
    c = cfg(B=2, H=2)
    small = torch.zeros(3, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dlb._check_step_tensors(c, small, small, small, torch.zeros(4), torch.zeros(4), None,
                                torch.zeros(512))
    with pytest.raises(TypeError):
        dlb._check_step_tensors(c, torch.zeros(512), torch.zeros(512), torch.zeros(512),
                                torch.zeros(4), torch.zeros(4), None, torch.zeros(512))
    # GDN-2: beta carries the erase gate [B,H,d_k], bonus the write gate [B,H,d_v]
    g = cfg(variant="gdn2", B=2, H=2, in_dtype="f32")
    ok = dict(q=torch.zeros(512), k=torch.zeros(512), v=torch.zeros(512), decay=torch.zeros(512),
              beta=torch.zeros(512), bonus=torch.zeros(512), o=torch.zeros(512))
    dlb._check_step_tensors(g, **ok)
    for name in ("beta", "bonus", "decay"):
        bad = dict(ok)
        bad[name] = torch.zeros(4)
        with pytest.raises(ValueError):
            dlb._check_step_tensors(g, **bad)


def test_load_seqs_checks_indices_on_the_host():
    c = cfg()
    h = dlb.dl_state_create(c, 0x100000, 0x200000, 0x300000)
    try:
        ld = dlb._lib.dl_state_load_seqs
        arr = lambda *x: (ctypes.c_int32 * len(x))(*x)
        assert ld(h, 2, arr(0, 0), None, None) == dlb.DL_ERR_ARG     # repeated
        assert ld(h, 1, arr(4), None, None) == dlb.DL_ERR_ARG        # out of range (B=4)
        assert ld(h, 1, arr(-1), None, None) == dlb.DL_ERR_ARG
        assert ld(h, -1, arr(0), None, None) == dlb.DL_ERR_ARG
        assert ld(h, 1, None, None, None) == dlb.DL_ERR_ARG
        assert ld(h, 1, arr(1), 0x1004, None) == dlb.DL_ERR_ALIGN
        assert ld(h, 0, None, None, None) == dlb.DL_OK                # nothing to do
    finally:
        dlb.dl_state_destroy(h)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_int8_code_swizzle_is_a_chunk_permutation(dk, dv):
    # logical (row, c) -> physical position: each row's 16-byte chunks are
    # permuted (XOR with row mod 8, or (row / 2) mod 4 for d_k = 64), bytes
    # inside a chunk stay in place, and eight consecutive rows put one logical
    # chunk into eight different 16-byte bank groups
    import torch
    st = object.__new__(dlb.DeltaLogState)
    st.cfg = cfg(d_k=dk, d_v=dv, base="q8")
    st.base = torch.empty(8)
    perm = st._q8_perm().view(dv, dk)
    assert sorted(perm.reshape(-1).tolist()) == list(range(dv * dk))
    assert torch.all(perm // dk == torch.arange(dv).view(dv, 1))
    assert torch.all(perm % 16 == torch.arange(dk).view(1, dk) % 16)
    groups = (perm[:8, ::16] // 16) % 8          # rows 0..7, each logical chunk
    for j in range(dk // 16):
        assert len(set(groups[:, j].tolist())) == 8


@pytest.mark.parametrize("variant", ["gdn", "kda", "gdn2", "rwkv6"])
@pytest.mark.parametrize("L", [1, 16, 48, 64])
@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
def test_q8_every_log_length_is_built(variant, L, fused, in_dtype):
    # the int8 merge takes the per-warp fold wherever its TMEM pipeline would
    # not fit in shared memory (long vector-decay logs), and the fused step
    # stages key fragments except for GDN with bf16 keys, so a state of every
    # L up to 64 can be created in both merge modes and for both key types
    # (host-side check of the kernels' shared memory, no launch)
    d = 64 if variant == "rwkv6" else 128
    c = cfg(variant=variant, d_k=d, d_v=d, L=L, base="q8", fused_merge=fused,
            in_dtype=in_dtype).c()
    st = ctypes.c_void_p()
    rc = dlb._lib.dl_state_create(ctypes.byref(c), ctypes.c_void_p(1 << 20), ctypes.c_void_p(2 << 20),
                                  ctypes.c_void_p(3 << 20), ctypes.byref(st))
    assert rc == dlb.DL_OK
    assert dlb._lib.dl_state_destroy(st) == dlb.DL_OK
