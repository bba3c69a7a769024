"""Host-side checks of the C ABI (no GPU needed).

The library links the CUDA runtime statically and opens the driver only on
its first CUDA call. It therefore loads on a host without a GPU. These tests
call only what returns before any CUDA call: status strings, the version,
the workspace size, and argument checks that reject their input. Fake device
pointers appear only in calls that a check rejects before any launch.
"""
import ctypes
import os
import re

import pytest

import learned_block_sparse_warp_b200 as sas
from learned_block_sparse_warp_b200 import Params, lib, sas_params

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
A = 0x7F0000000000  # aligned fake address; only ever handed to calls that reject their arguments


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"SAS_API\s+[\w\s\*]+?\b(sas_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert {"sas_topk_select", "sas_gate_lse", "sas_fwd", "sas_bwd", "sas_bwd_workspace_size",
            "sas_bwd_workspace_size_min", "sas_decode",
            "sas_decode_combine", "sas_get_device_error", "sas_status_string", "sas_version"} <= names
    raw = ctypes.CDLL(sas.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_status_strings_and_version():
    for code, name in sas.STATUS.items():
        assert sas.sas_status_string(code).startswith(name)
    assert "unknown" in sas.sas_status_string(99)
    assert sas.sas_version() >= 100


def _p(**kw):
    base = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, seq_len=1024, top_k=4)
    base.update(kw)
    return Params(**base)


def _fwd(p, q=A, k=A, v=A, s=A, idx=A, lse_s=A, o=A, lse_o=None):
    c = p.c() if p is not None else None
    return lib.sas_fwd(ctypes.byref(c) if c is not None else None, q, k, v, s, idx, lse_s, o, lse_o, None)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), UNSUPPORTED),
    (dict(head_dim=256), UNSUPPORTED),
    (dict(block=32), UNSUPPORTED),
    (dict(seq_len=1000), INVALID),
    (dict(seq_len=0), INVALID),
    (dict(n_q_heads=3), INVALID),
    (dict(top_k=0), INVALID),
    (dict(top_k=2049), INVALID),
    (dict(seq_len=64 * (2 ** 19 + 1), n_q_heads=1, n_kv_heads=1), UNSUPPORTED),
    (dict(batch=0), INVALID),
    (dict(gate_mode=7), INVALID),
    (dict(softmax_scale=-1.0), INVALID),
    (dict(softmax_scale=float("nan")), INVALID),
])
def test_fwd_rejects_bad_params(kw, code):
    assert _fwd(_p(**kw)) == code


def test_null_params_and_pointers():
    assert _fwd(None) == INVALID
    assert _fwd(_p(), q=None) == INVALID
    assert _fwd(_p(), idx=None) == INVALID
    assert _fwd(_p(), o=None) == INVALID
    # gated needs s and lse_s
    assert _fwd(_p(), s=None) == INVALID
    assert _fwd(_p(), lse_s=None) == INVALID


def test_misaligned_pointers_rejected():
    assert _fwd(_p(), q=A + 2) == INVALID
    assert _fwd(_p(), lse_o=A + 4) == INVALID
    c = _p().c()
    assert lib.sas_topk_select(ctypes.byref(c), A + 8, None, A, None, None) == INVALID
    assert lib.sas_topk_select(ctypes.byref(c), A, None, None, None, None) == INVALID
    assert lib.sas_gate_lse(ctypes.byref(c), A, None, None, None) == INVALID


def test_workspace_size_and_check():
    p = _p(batch=2, n_q_heads=8, n_kv_heads=2, seq_len=2048, top_k=8)
    n_min = sas.sas_bwd_workspace_size_min(p)
    n = sas.sas_bwd_workspace_size(p)
    B, Hq, Hkv, N, d, NB, K = 2, 8, 2, 2048, 128, 32, 8
    # D rows, dl, the reverse index (counts, offsets, entries, gates) and the selection bitmap with
    # its per-word prefix counts (one word each per 32 blocks and row); no fp32 dQ at d = 128
    W = (NB + 31) // 32
    lower = 4 * (B * Hq * N + B * Hkv * NB * K) + 4 * (B * Hkv * NB * 2 + 2 * B * Hkv * NB * K) \
        + 8 * B * Hkv * NB * W
    assert lower <= n_min <= lower + 9 * 256
    # the full size adds one 16 KB dZ tile per (batch, KV head, query block, attended block, head pair)
    tiles = B * Hkv * sum(1 + min(K, t) for t in range(NB)) * ((Hq // Hkv + 1) // 2)
    assert n_min + tiles * 16384 <= n <= n_min + tiles * 16384 + 256
    c = p.c()
    args = [A] * 13
    # too small, unaligned, or missing workspace: SAS_ERR_WORKSPACE before any launch
    assert lib.sas_bwd(ctypes.byref(c), *args, A, n_min - 1, None) == WORKSPACE
    assert lib.sas_bwd(ctypes.byref(c), *args, A + 16, n, None) == WORKSPACE
    assert lib.sas_bwd(ctypes.byref(c), *args, None, n, None) == WORKSPACE
    size = ctypes.c_size_t(0)
    for fn in (lib.sas_bwd_workspace_size, lib.sas_bwd_workspace_size_min):
        assert fn(None, ctypes.byref(size)) == INVALID
        assert fn(ctypes.byref(c), None) == INVALID


def test_workspace_d64_has_both_forms():
    # the same tcgen05 passes serve d = 64: the full workspace adds the same dZ tiles (128 x 64 bf16
    # per query block, attended block and head pair, independent of d)
    p, p128 = _p(head_dim=64), _p(head_dim=128)
    extra64 = sas.sas_bwd_workspace_size(p) - sas.sas_bwd_workspace_size_min(p)
    extra128 = sas.sas_bwd_workspace_size(p128) - sas.sas_bwd_workspace_size_min(p128)
    assert extra64 == extra128 > 0


def test_decode_split_count_checked():
    c = _p(top_k=4).c()
    base = [A, A, A, A, A, A, A]
    assert lib.sas_decode(ctypes.byref(c), *base, 0, A, A, None) == INVALID
    assert lib.sas_decode(ctypes.byref(c), *base, 6, A, A, None) == INVALID  # > K + 1
    assert lib.sas_decode_combine(ctypes.byref(c), 0, A, A, A, None, None) == INVALID
    c16 = _p(n_q_heads=32, n_kv_heads=2).c()  # G = 16: no decode kernel
    assert lib.sas_decode(ctypes.byref(c16), *base, 2, A, A, None) == UNSUPPORTED


def test_params_struct_layout():
    assert ctypes.sizeof(sas_params) == 9 * 4
    assert [f[0] for f in sas_params._fields_] == ["batch", "n_q_heads", "n_kv_heads", "head_dim", "seq_len",
                                                    "block", "top_k", "softmax_scale", "gate_mode"]
    hdr = open(os.path.join(ROOT, "include", "sas.h")).read()
    body = hdr[hdr.index("typedef struct {"):hdr.index("} sas_params;")]
    assert re.findall(r"(?:int|float)\s+(\w+);", body) == [f[0] for f in sas_params._fields_]


def test_python_binding_refuses_cpu_tensors():
    import torch
    p = _p(seq_len=128, top_k=1, n_q_heads=2, n_kv_heads=2, head_dim=64)
    s = torch.zeros(1, 2, 2, 2)
    idx = torch.zeros(1, 2, 2, 1, dtype=torch.int32)
    with pytest.raises(ValueError):
        sas.sas_topk_select(p, s, idx)


def test_decode_paged_checked():
    c = _p(top_k=4).c()

    def call(n_pages=8, table=A, n_split=2, params=c):
        # p, q, k_pages, v_pages, n_pages, block_table, cache_len, s, idx, lse_s, n_split, o_part, lse_part, stream
        return lib.sas_decode_paged(ctypes.byref(params), A, A, A, n_pages, table, A, A, A, A, n_split, A, A, None)

    assert call(n_pages=0) == INVALID
    assert call(n_pages=-3) == INVALID
    assert call(n_pages=1 << 30) == INVALID  # page rows would overflow a 32-bit row index
    assert call(table=None) == INVALID
    assert call(n_split=0) == INVALID
    assert call(n_split=6) == INVALID  # > K + 1
    c16 = _p(n_q_heads=32, n_kv_heads=2).c()  # G = 16: no decode kernel
    assert call(params=c16) == UNSUPPORTED


def test_gate_ablation_inputs_checked():
    # the ablations read s but not lse_s: s is required, lse_s may be NULL
    for mode in (2, 3):
        assert _fwd(_p(gate_mode=mode), s=None) == INVALID
    assert _fwd(_p(gate_mode=0), lse_s=None) == INVALID
    # the gate outside the softmax is softmax-normalised: it needs s and lse_s
    assert _fwd(_p(gate_mode=4), s=None) == INVALID
    assert _fwd(_p(gate_mode=4), lse_s=None) == INVALID
    assert _fwd(_p(gate_mode=5)) == INVALID
    c = _p(gate_mode=2).c()
    assert lib.sas_decode(ctypes.byref(c), A, A, A, A, None, A, None, 2, A, A, None) == INVALID  # s missing


def test_decode_split_size_limited():
    # a split may cover at most 64 blocks: K = 256 needs n_split >= 5
    c = _p(top_k=256, seq_len=32768).c()
    base = [A, A, A, A, A, A, A]
    assert lib.sas_decode(ctypes.byref(c), *base, 1, A, A, None) == UNSUPPORTED
    assert lib.sas_decode(ctypes.byref(c), *base, 4, A, A, None) == UNSUPPORTED
    assert lib.sas_decode_paged(ctypes.byref(c), A, A, A, 8, A, A, A, A, A, 4, A, A, None) == UNSUPPORTED


def test_decode_fused_checked():
    # p, q, kc, vc, cache_len, s, idx, lse_s, o, lse_o, stream
    def call(params, s=A, o=A, idx=A, cl=A):
        return lib.sas_decode_fused(ctypes.byref(params), A, A, A, cl, s, idx, A, o, A, None)

    c = _p(top_k=16, seq_len=32768).c()
    assert call(c, s=None) == INVALID  # the scores drive the selection
    assert call(c, o=None) == INVALID
    assert call(c, cl=None) == INVALID
    assert call(c, idx=A + 4) == INVALID  # misaligned optional output
    assert call(_p(top_k=256, seq_len=32768).c()) == UNSUPPORTED  # the picks live in shared memory
    assert call(_p(top_k=16, seq_len=64 * 4096).c()) == UNSUPPORTED  # so do the row's keys
    assert call(_p(n_q_heads=32, n_kv_heads=2).c()) == UNSUPPORTED  # G = 16
    paged = lib.sas_decode_fused_paged
    # p, q, k_pages, v_pages, n_pages, table, cache_len, s, idx, lse_s, o, lse_o, stream
    assert paged(ctypes.byref(c), A, A, A, 0, A, A, A, A, A, A, A, None) == INVALID
    assert paged(ctypes.byref(c), A, A, A, 8, None, A, A, A, A, A, A, None) == INVALID
    assert paged(ctypes.byref(c), A, A, A, 1 << 30, A, A, A, A, A, A, A, None) == INVALID


def test_block_mean_keys_checked():
    c = _p().c()
    f = lib.sas_block_mean_keys
    assert f(None, A, None, A, None) == INVALID
    assert f(ctypes.byref(c), None, None, A, None) == INVALID
    assert f(ctypes.byref(c), A, None, None, None) == INVALID
    assert f(ctypes.byref(c), A + 2, None, A, None) == INVALID
    assert f(ctypes.byref(c), A, A + 4, A, None) == INVALID  # cache_len misaligned
    assert f(ctypes.byref(_p(head_dim=96).c()), A, None, A, None) == UNSUPPORTED


def test_decode_select_scored_checked():
    c = _p().c()

    def call(params=c, q=A, kmean=A, cl=A, s=A, idx=A, lse=None):
        return lib.sas_decode_select_scored(ctypes.byref(params) if params is not None else None, q, kmean, cl, s,
                                            idx, lse, None)

    assert call(params=None) == INVALID
    for kw in ("q", "kmean", "cl", "s", "idx"):
        assert call(**{kw: None}) == INVALID, kw
    assert call(lse=A + 4) == INVALID
    assert call(params=_p(head_dim=96).c()) == UNSUPPORTED
    # a row of more than 8 x 53,248 history blocks does not fit a cluster's shared memory
    big = _p(n_q_heads=1, n_kv_heads=1, seq_len=64 * (8 * 53248 + 2)).c()
    assert call(params=big) == UNSUPPORTED


def test_host_step_structs_match_the_header():
    """Field order and size of sas_host_step / sas_device_slot, compiled from the header by gcc."""
    import subprocess
    import tempfile
    src = r'''
#include <stddef.h>
#include <stdio.h>
#include "sas.h"
#define F(T, m) printf("%s %zu\n", #m, offsetof(T, m));
int main(void) {
  printf("host %zu\n", sizeof(sas_host_step));
  F(sas_host_step, q) F(sas_host_step, k) F(sas_host_step, v) F(sas_host_step, s) F(sas_host_step, dO)
  F(sas_host_step, o) F(sas_host_step, lse_o) F(sas_host_step, dq) F(sas_host_step, dk) F(sas_host_step, dv)
  F(sas_host_step, ds)
  printf("slot %zu\n", sizeof(sas_device_slot));
  F(sas_device_slot, q) F(sas_device_slot, k) F(sas_device_slot, v) F(sas_device_slot, dO) F(sas_device_slot, o)
  F(sas_device_slot, dq) F(sas_device_slot, dk) F(sas_device_slot, dv) F(sas_device_slot, s)
  F(sas_device_slot, lse_s) F(sas_device_slot, lse_o) F(sas_device_slot, ds) F(sas_device_slot, idx)
  F(sas_device_slot, ws) F(sas_device_slot, ws_bytes)
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "layout.c")
        exe = os.path.join(tmp, "layout")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-std=c11", f"-I{os.path.join(ROOT, 'include')}", c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(ln.split() for ln in lines if ln)
    assert int(got["host"]) == ctypes.sizeof(sas.sas_host_step)
    assert int(got["slot"]) == ctypes.sizeof(sas.sas_device_slot)
    host_off = [getattr(sas.sas_host_step, n).offset for n, _ in sas.sas_host_step._fields_]
    slot_off = [getattr(sas.sas_device_slot, n).offset for n, _ in sas.sas_device_slot._fields_]
    vals = [int(v) for k, v in (ln.split() for ln in lines if ln) if k not in ("host", "slot")]
    assert vals == host_off + slot_off


def test_train_steps_host_checked():
    p = _p()
    c = p.c()
    n = sas.sas_bwd_workspace_size(p)
    slot = sas.sas_device_slot(*([A] * 14), n)
    step = sas.sas_host_step(*([A] * 11))
    slots = (sas.sas_device_slot * 2)(slot, slot)
    steps = (sas.sas_host_step * 3)(step, step, step)
    f = lib.sas_train_steps_host
    assert f(None, 3, steps, slots, None) == INVALID
    assert f(ctypes.byref(c), 0, steps, slots, None) == INVALID
    assert f(ctypes.byref(c), 3, None, slots, None) == INVALID
    assert f(ctypes.byref(c), 3, steps, None, None) == INVALID
    n_min = sas.sas_bwd_workspace_size_min(p)
    small = (sas.sas_device_slot * 2)(slot, sas.sas_device_slot(*([A] * 14), n_min - 1))
    assert f(ctypes.byref(c), 3, steps, small, None) == WORKSPACE
    bad_slot = (sas.sas_device_slot * 2)(slot, sas.sas_device_slot(*([A] * 13), None, n))
    assert f(ctypes.byref(c), 3, steps, bad_slot, None) == WORKSPACE
    no_dq = sas.sas_device_slot(*([A] * 14), n)
    no_dq.dq = None
    assert f(ctypes.byref(c), 3, steps, (sas.sas_device_slot * 2)(slot, no_dq), None) == INVALID
    bad_step = sas.sas_host_step(*([A] * 11))
    bad_step.dO = None
    assert f(ctypes.byref(c), 3, (sas.sas_host_step * 3)(step, step, bad_step), slots, None) == INVALID
    # no ds without a gate
    c_none = _p(gate_mode=1).c()
    assert f(ctypes.byref(c_none), 3, steps, slots, None) == INVALID


def test_plain_c_program_links_the_library():
    """The boundary is usable from C alone: compile against include/sas.h, link libsas_b200.so and
    call the entry points that need no GPU (version, status strings, workspace size, argument checks)."""
    import subprocess
    import tempfile
    src = r'''
#include <stdio.h>
#include "sas.h"
int main(void) {
  sas_params p = {1, 8, 2, 128, 1024, 64, 4, 0.0f, SAS_GATE_LOG_SOFTMAX};
  size_t ws = 0;
  if (sas_bwd_workspace_size(&p, &ws) != SAS_OK || ws == 0) return 1;
  if (sas_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != SAS_ERR_INVALID_ARG) return 2;
  p.head_dim = 96;
  if (sas_bwd_workspace_size(&p, &ws) != SAS_ERR_UNSUPPORTED) return 3;
  printf("%d %zu %s\n", sas_version(), ws, sas_status_string(SAS_ERR_TIMEOUT));
  return 0;
}
'''
    lib_dir = os.path.dirname(sas.LIB_PATH)
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "use_sas.c")
        exe = os.path.join(tmp, "use_sas")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-std=c11", f"-I{os.path.join(ROOT, 'include')}", c, f"-L{lib_dir}", "-l:libsas_b200.so",
                        f"-Wl,-rpath,{lib_dir}", "-o", exe], check=True)
        r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    ver, ws, msg = r.stdout.split(maxsplit=2)
    assert int(ver) == sas.sas_version() and int(ws) == sas.sas_bwd_workspace_size(_p(n_q_heads=8, n_kv_heads=2))
    assert msg.startswith("SAS_ERR_TIMEOUT")
