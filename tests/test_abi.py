"""The C-ABI library loads, exports every declared symbol, and rejects bad arguments
on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_62_b200 import kda as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", txt)
    return sorted(set(names))


def test_header_declares_expected_entry_points():
    names = declared_symbols()
    for must in ["kda_prefill", "kda_prefill_workspace_size", "kda_decode_step", "kda_status_string",
                 "kda_last_error", "kda_read_device_status"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(K.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(L, n)]
    assert not missing, missing
    # and the binding knows every one of them
    assert set(declared_symbols()) <= set(K.SIGNATURES)


def test_status_strings():
    L = K.lib()
    assert L.kda_status_string(0) == b"KDA_OK"
    assert L.kda_status_string(4) == b"KDA_ERR_TIMEOUT"
    assert L.kda_status_string(99) == b"KDA_ERR_UNKNOWN"
    assert L.kda_version() >= 100


def test_workspace_size():
    assert K.workspace_size(1, 64, 2, 32, 32, torch.float32) >= 256
    assert K.workspace_size(24, 10**6, 32, 128, 128, torch.bfloat16) % 256 == 0
    L = K.lib()
    assert L.kda_prefill_workspace_size(1, 10, 2, 48, 32, 0) == 0  # unsupported d_k
    assert L.kda_prefill_workspace_size(1, 10, 0, 32, 32, 0) == 0


def _prefill_raw(**over):
    """Call kda_prefill with fake (never dereferenced) pointers; validation fails first."""
    L = K.lib()
    cu = (ctypes.c_int32 * 3)(*over.pop("cu", [0, 5, 9]))
    fake = ctypes.c_void_p(0x10000)
    a = dict(q=fake, k=fake, v=fake, la=fake, beta=fake, s0=None, cud=fake, cuh=cu, N=2, T=9, H=2,
             dk=32, dv=32, dt=0, out=ctypes.c_void_p(0x20000), fs=None, ws=None, wsb=0, st=None)
    a.update(over)
    rc = L.kda_prefill(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["cud"],
                       ctypes.cast(a["cuh"], ctypes.c_void_p), a["N"], a["T"], a["H"], a["dk"],
                       a["dv"], a["dt"], a["out"], a["fs"], a["ws"], a["wsb"], a["st"])
    return rc, L.kda_last_error().decode()


@pytest.mark.parametrize("over,needle", [
    (dict(H=0), "H=0"),
    (dict(dk=48), "d_k=48"),
    (dict(dv=256), "d_v=256"),
    (dict(dt=7), "dtype"),
    (dict(N=-1), "num_seqs"),
    (dict(cu=[1, 5, 9]), "cu_seqlens[0]"),
    (dict(cu=[0, 5, 4], T=4), "decreases"),
    (dict(T=10), "total_tokens"),
    (dict(q=None), "required"),
    (dict(cud=None), "cu_seqlens_dev"),
    (dict(q=ctypes.c_void_p(0x10004)), "16-byte"),
    (dict(out=ctypes.c_void_p(0x10000)), "alias"),
    (dict(), "workspace"),  # all else valid: the missing workspace is reported
    (dict(ws=ctypes.c_void_p(0x30000), wsb=16), "workspace"),
    (dict(ws=ctypes.c_void_p(0x30010), wsb=1 << 20), "256-byte"),
])
def test_prefill_rejects_bad_arguments(over, needle):
    rc, msg = _prefill_raw(**over)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT
    assert needle in msg, msg


def test_decode_rejects_bad_arguments():
    L = K.lib()
    fake = ctypes.c_void_p(0x10000)
    rc = L.kda_decode_step(fake, fake, fake, fake, fake, fake, 4, 2, 64, 100, 1,
                           ctypes.c_void_p(0x20000), None, 0, None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and b"d_v=100" in L.kda_last_error()
    rc = L.kda_decode_step(fake, fake, fake, fake, fake, None, 4, 2, 64, 64, 1,
                           ctypes.c_void_p(0x20000), None, 0, None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and b"required" in L.kda_last_error()
    # zero sequences: a no-op that needs no pointers
    assert L.kda_decode_step(None, None, None, None, None, None, 0, 2, 64, 64, 1, None, None, 0,
                             None) == K.KDA_OK


def test_zero_sequences_is_a_noop():
    L = K.lib()
    rc = L.kda_prefill(None, None, None, None, None, None, None, None, 0, 0, 4, 128, 128, 1, None,
                       None, None, 0, None)
    assert rc == K.KDA_OK


def test_binding_requires_cuda_tensors():
    x = torch.zeros(4, 2, 32)
    with pytest.raises(ValueError, match="CUDA"):
        K.prefill(x, x, x, x, torch.zeros(4, 2))


def test_product_path_does_not_import_oracle():
    """The library binding and package never import the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "gated_delta_rule_62_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert not re.search(r"^\s*(from|import)\s+oracle", src, re.M), fn


def test_slot_entry_points_reject_bad_arguments():
    L = K.lib()
    fake = ctypes.c_void_p(0x10000)
    out = ctypes.c_void_p(0x20000)
    cu = (ctypes.c_int32 * 3)(0, 5, 9)
    cuh = ctypes.cast(cu, ctypes.c_void_p)

    def prefill_slots(pool=fake, slots=4, init=fake, fin=fake, ws=None, wsb=0):
        rc = L.kda_prefill_slots(fake, fake, fake, fake, fake, pool, slots, init, fin, fake, cuh, 2,
                                 9, 2, 32, 32, 0, out, ws, wsb, None)
        return rc, L.kda_last_error().decode()

    rc, msg = prefill_slots(pool=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "state_pool" in msg
    rc, msg = prefill_slots(slots=-1)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "pool_slots" in msg
    rc, msg = prefill_slots(init=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "init_slot_dev" in msg
    rc, msg = prefill_slots()  # all else valid: the missing workspace is reported
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "workspace" in msg

    def decode_slots(slot=fake, ws=None, wsb=0, pool=fake, slots=4):
        rc = L.kda_decode_step_slots(fake, fake, fake, fake, fake, pool, slots, slot, 4, 2, 64, 64, 1,
                                     out, ws, wsb, None)
        return rc, L.kda_last_error().decode()

    rc, msg = decode_slots(slot=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "slot_dev" in msg
    rc, msg = decode_slots()
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "workspace" in msg
    rc, msg = decode_slots(ws=ctypes.c_void_p(0x30010), wsb=256)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "256-byte aligned" in msg
    rc, msg = decode_slots(pool=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "state_pool" in msg
    # zero sequences: a no-op
    assert L.kda_decode_step_slots(None, None, None, None, None, None, 0, None, 0, 2, 64, 64, 1, None,
                                   None, 0, None) == K.KDA_OK


def test_speculative_entry_points_reject_bad_arguments():
    L = K.lib()
    fake = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x40000)

    def verify(T=4, state=fake, slot=None, slots=0, ws=ws, wsb=256, out=ctypes.c_void_p(0x20000),
               u=ctypes.c_void_p(0x30000)):
        rc = L.kda_decode_verify(fake, fake, fake, fake, fake, state, slots, slot, 3, T, 2, 64, 64, 1,
                                 out, u, ws, wsb, None)
        return rc, L.kda_last_error().decode()

    for T in (0, K.MAX_DRAFT_TOKENS + 1):
        rc, msg = verify(T=T)
        assert rc == K.KDA_ERR_INVALID_ARGUMENT and "T=" in msg
    rc, msg = verify(state=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "state" in msg
    rc, msg = verify(slot=fake, slots=-2)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "pool_slots" in msg
    rc, msg = verify(ws=None, wsb=0)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "workspace" in msg
    rc, msg = verify(u=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "u_cache" in msg
    rc, msg = verify(out=fake)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "alias" in msg
    rc, msg = verify(u=ctypes.c_void_p(0x20000))
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "alias" in msg

    def commit(acc=fake, T=4, state=ctypes.c_void_p(0x50000), u=ctypes.c_void_p(0x30000)):
        rc = L.kda_decode_commit(fake, fake, u, state, 0, None, acc, 3, T, 2, 64, 64, 1, ws, 256, None)
        return rc, L.kda_last_error().decode()

    rc, msg = commit(acc=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "accepted_dev" in msg
    rc, msg = commit(T=17)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "T=" in msg
    rc, msg = commit(u=ctypes.c_void_p(0x50000))
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "aliases the state" in msg
    # zero sequences: no-ops
    assert L.kda_decode_verify(None, None, None, None, None, None, 0, None, 0, 4, 2, 64, 64, 1, None,
                               None, ws, 256, None) == K.KDA_OK
    assert L.kda_decode_commit(None, None, None, None, 0, None, None, 0, 4, 2, 64, 64, 1, ws, 256,
                               None) == K.KDA_OK


def test_max_draft_tokens_matches_header():
    txt = open(os.path.join(ROOT, "include", "kda.h")).read()
    assert int(re.search(r"#define KDA_MAX_DRAFT_TOKENS (\d+)", txt).group(1)) == K.MAX_DRAFT_TOKENS


def test_commit_verify_rejects_bad_arguments():
    L = K.lib()
    fake = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x40000)
    out, u, pu = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), ctypes.c_void_p(0x60000)
    state = ctypes.c_void_p(0x50000)

    def cv(Tp=4, acc=fake, out=out, u=u, pu=pu, pk=fake):
        rc = L.kda_decode_commit_verify(pk, fake, pu, acc, Tp, fake, fake, fake, fake, fake, state, 0,
                                        None, 3, 4, 2, 64, 64, 1, out, u, ws, 256, None)
        return rc, L.kda_last_error().decode()

    for Tp in (0, K.MAX_DRAFT_TOKENS + 1):
        rc, msg = cv(Tp=Tp)
        assert rc == K.KDA_ERR_INVALID_ARGUMENT and "T_prev" in msg
    rc, msg = cv(acc=None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "accepted_dev" in msg
    rc, msg = cv(u=pu)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "previous draft" in msg
    rc, msg = cv(pk=out)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "previous draft" in msg


def test_prologue_entry_point_rejects_bad_arguments():
    L = K.lib()
    fake = ctypes.c_void_p(0x10000)
    cu = (ctypes.c_int32 * 2)(0, 5)
    cuh = ctypes.cast(cu, ctypes.c_void_p)

    def call(flags, scale):
        rc = L.kda_prefill_prologue(fake, fake, fake, fake, fake, None, fake, cuh, 1, 5, 2, 32, 32, 0,
                                    ctypes.c_void_p(0x20000), None, None, 0, flags, scale, None)
        return rc, L.kda_last_error().decode()

    rc, msg = call(8, 1.0)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "unknown bits" in msg
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        rc, msg = call(K.PROLOGUE_GATE_SOFTPLUS, bad)
        assert rc == K.KDA_ERR_INVALID_ARGUMENT and "gate_scale" in msg
    rc, msg = call(K.PROLOGUE_ALL, 1.0 / 16)  # valid up to the missing workspace
    assert rc == K.KDA_ERR_INVALID_ARGUMENT and "workspace" in msg


def test_prologue_flags_match_header():
    txt = open(os.path.join(ROOT, "include", "kda.h")).read()
    got = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define KDA_PROLOGUE_(\w+) (\d+)u", txt)}
    assert got == {"QK_L2NORM": K.PROLOGUE_QK_L2NORM, "GATE_SOFTPLUS": K.PROLOGUE_GATE_SOFTPLUS,
                   "BETA_SIGMOID": K.PROLOGUE_BETA_SIGMOID}
    import oracle
    assert (oracle.QK_L2NORM, oracle.GATE_SOFTPLUS, oracle.BETA_SIGMOID) == (1, 2, 4)
