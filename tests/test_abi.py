"""The C ABI library: it builds, loads, exports every symbol that include/kda.h declares, and
rejects bad arguments on the host before touching a GPU.  CPU only (no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

import __graft_entry__  # noqa: E402

__graft_entry__._builder().build()
import kda_chunkwise_b200 as kda  # noqa: E402

lib = kda.lib


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size",
                 "kda_chunk_fwd_workspace_min", "kda_status_string", "kda_sync_check",
                 "kda_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    raw = ctypes.CDLL(kda.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"libkda.so does not export {name}"


def test_status_strings():
    for code in range(6):
        assert kda.kda_status_string(code) != "unknown status"
    assert kda.kda_status_string(0) == "ok"
    assert kda.kda_status_string(kda.KDA_ERR_RANGE) == "value outside the fp16 operand range"


def test_workspace_sizes():
    mn = kda.kda_chunk_fwd_workspace_min(8192, 1, 8192, 32, 128, 128)
    rec = kda.kda_chunk_fwd_workspace_size(8192, 1, 8192, 32, 128, 128)
    assert 0 < mn <= rec
    assert rec % 256 == 0 and mn % 256 == 0
    assert kda.kda_chunk_fwd_workspace_size(8192, 1, 8192, 32, 96, 128) == 0   # unsupported d_k
    assert kda.kda_chunk_fwd_workspace_size(-1, 1, 0, 32, 128, 128) == 0
    # a short batch never asks for more than its own chunks
    small = kda.kda_chunk_fwd_workspace_size(64, 1, 64, 2, 64, 64)
    assert small == kda.kda_chunk_fwd_workspace_min(64, 1, 64, 2, 64, 64)


def test_prefill_kernel_choice_by_units():
    # The cluster kernel (1) while its units need at most two waves of four-CTA clusters, the
    # per-unit kernel (2) beyond: one switch, at twice the clusters that fit at once.  A 148-SM
    # B200 holds 33 (the occupancy query; 33 is also the library's figure for 148 SMs when it
    # cannot query a device), so the switch is after 66 units; a cluster must sit inside one GPC,
    # so the figure lies below a quarter of the SM count.
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    paths = [kda.kda_prefill_path(u, 128, 128) for u in range(1, 4 * sms + 1)]
    edge = paths.index(2)   # units <= edge run the cluster kernel
    assert set(paths[:edge]) == {1} and set(paths[edge:]) == {2}
    assert edge % 2 == 0 and 2 <= edge <= 2 * (sms // 4)
    if not torch.cuda.is_available():
        assert edge == 66
    assert kda.kda_prefill_path(4096, 64, 128) == 1      # other head sizes: the cluster kernel only
    kda.kda_set_prefill_path(2)
    try:
        assert kda.kda_prefill_path(1, 128, 128) == 2
        assert kda.kda_chunk_fwd_workspace_min(8192, 1, 8192, 32, 128, 128) == 0
    finally:
        kda.kda_set_prefill_path(0)


def _fwd(**over):
    base = dict(q=16, k=16, v=16, a=16, beta=16, gate=None, A_log=16, cu=16, N=1, T=64,
                max_seqlen=64, H=2, dk=64, dv=64, scale=1.0, S0=None, SF=None, out=16,
                out_dtype=0, ws=256, ws_bytes=1 << 30, stream=None)
    base.update(over)
    b = base
    return lib.kda_chunk_fwd(b["q"], b["k"], b["v"], b["a"], b["beta"], b["gate"], b["A_log"],
                             b["cu"], b["N"], b["T"], b["max_seqlen"], b["H"], b["dk"], b["dv"],
                             b["scale"], b["S0"], b["SF"], b["out"], b["out_dtype"], b["ws"],
                             b["ws_bytes"], b["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(cu=None), kda.KDA_ERR_INVALID_ARG),
    (dict(q=24), kda.KDA_ERR_INVALID_ARG),          # misaligned
    (dict(beta=18), kda.KDA_ERR_INVALID_ARG),       # beta needs 4-byte alignment
    (dict(out_dtype=7), kda.KDA_ERR_INVALID_ARG),
    (dict(ws=None), kda.KDA_ERR_INVALID_ARG),
    (dict(ws=16 + 256), kda.KDA_ERR_INVALID_ARG),   # workspace must be 256-byte aligned
    (dict(ws_bytes=1024), kda.KDA_ERR_INVALID_ARG),  # too small
    (dict(N=0, T=5), kda.KDA_ERR_INVALID_ARG),
])
def test_chunk_fwd_rejects_bad_arguments(over, code):
    assert _fwd(**over) == code
    assert lib.kda_last_error().decode()


def test_chunk_fwd_empty_batch_is_ok():
    assert _fwd(N=0, T=0) == kda.KDA_OK
    assert _fwd(N=0, T=0, beta=20) == kda.KDA_OK   # 4-byte aligned beta is enough


def test_decode_rejects_bad_arguments():
    f = lib.kda_decode_step
    assert f(16, 16, 16, 16, 16, None, 16, 16, 16, 0, 4, 0, 128, 128, 1.0, None) == kda.KDA_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, None, 16, 16, 16, 0, 4, 2, 128, 80, 1.0, None) == kda.KDA_ERR_UNSUPPORTED
    assert f(None, 16, 16, 16, 16, None, 16, 16, 16, 0, 4, 2, 128, 128, 1.0, None) == kda.KDA_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, 8, 16, 16, 16, 0, 4, 2, 128, 128, 1.0, None) == kda.KDA_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, None, 16, 16, 16, 5, 4, 2, 128, 128, 1.0, None) == kda.KDA_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, None, 16, 16, 16, 0, 0, 2, 128, 128, 1.0, None) == kda.KDA_OK


def test_inject_stall_validates_its_limit_on_the_host():
    assert lib.kda_inject_stall(1, 10) == kda.KDA_ERR_INVALID_ARG          # below 1 ms
    assert lib.kda_inject_stall(1, 5_000_000_000) == kda.KDA_ERR_INVALID_ARG   # above 4 s
    assert lib.kda_inject_stall(0, 0) == kda.KDA_OK
    with pytest.raises(kda.KDAError):
        kda.kda_inject_stall(True, 0)


def test_verify_and_commit_reject_bad_arguments():
    V, C = lib.kda_decode_verify, lib.kda_decode_commit
    ok = dict(q=16, k=16, v=16, a=16, beta=16, gate=None, A_log=16, state=16, u=16, out=16, dt=0, N=2, K=4,
              H=2, dk=128, dv=128)

    def ver(**o):
        a = dict(ok, **o)
        return V(a["q"], a["k"], a["v"], a["a"], a["beta"], a["gate"], a["A_log"], a["state"], a["u"], a["out"],
                 a["dt"], a["N"], a["K"], a["H"], a["dk"], a["dv"], 1.0, None)

    assert ver(K=0) == kda.KDA_ERR_INVALID_ARG
    assert ver(K=17) == kda.KDA_ERR_INVALID_ARG
    assert ver(dv=96) == kda.KDA_ERR_UNSUPPORTED
    assert ver(u=None) == kda.KDA_ERR_INVALID_ARG
    assert ver(q=8) == kda.KDA_ERR_INVALID_ARG          # misaligned
    assert ver(dt=5) == kda.KDA_ERR_INVALID_ARG
    assert ver(N=0) == kda.KDA_OK
    assert C(16, 16, 16, 16, 16, 16, 2, 0, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG       # K = 0
    assert C(16, 16, 16, None, 16, 16, 2, 4, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG     # accepted
    assert C(16, 16, 16, 18, 16, 16, 2, 4, 2, 128, 128, None) == kda.KDA_ERR_INVALID_ARG       # alignment
    assert C(16, 16, 16, 16, 16, 16, 0, 4, 2, 128, 128, None) == kda.KDA_OK


def test_short_conv_and_norm_gate_reject_bad_arguments():
    SC, NG = lib.kda_short_conv, lib.kda_output_norm_gate
    assert SC(16, 16, 16, 2, 64, 2, 128, 0, 1, 32, None) == kda.KDA_ERR_INVALID_ARG      # width 0
    assert SC(16, 16, 16, 2, 64, 2, 128, 5, 1, 32, None) == kda.KDA_ERR_INVALID_ARG      # width 5
    assert SC(16, 16, 16, 2, 64, 2, 80, 4, 1, 32, None) == kda.KDA_ERR_UNSUPPORTED       # d
    assert SC(16, 16, None, 2, 64, 2, 128, 4, 1, 32, None) == kda.KDA_ERR_INVALID_ARG    # cu_seqlens
    assert SC(8, 16, 16, 2, 64, 2, 128, 4, 1, 32, None) == kda.KDA_ERR_INVALID_ARG       # misaligned x
    assert SC(16, 16, 16, 0, 64, 2, 128, 4, 1, 32, None) == kda.KDA_ERR_INVALID_ARG      # tokens, no sequences
    assert SC(16, 16, 16, 2, 0, 2, 128, 4, 1, 32, None) == kda.KDA_OK                    # nothing to do
    assert NG(16, None, 16, 64, 2, 96, 1e-6, 32, 0, None) == kda.KDA_ERR_UNSUPPORTED
    assert NG(16, None, 16, 64, 2, 128, -1.0, 32, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert NG(16, None, None, 64, 2, 128, 1e-6, 32, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert NG(16, None, 16, 64, 2, 128, 1e-6, 32, 7, None) == kda.KDA_ERR_INVALID_ARG
    assert NG(16, None, 16, 0, 2, 128, 1e-6, 32, 0, None) == kda.KDA_OK


@pytest.mark.parametrize("entry", ["kda_chunk_bwd", "kda_chunk_bwd_chunkwise"])
def test_chunk_bwd_rejects_bad_arguments(entry):
    B = getattr(lib, entry)
    ok = dict(q=16, k=16, v=16, a=16, beta=16, gate=None, A_log=16, cu=16, N=1, T=64, H=2, dk=128, dv=128,
              S0=None, dout=16, dST=None, dq=16, dkk=16, dvv=16, da=16, db=16, dg=None, dA=16, dS0=None,
              ws=256, wsb=1 << 30)

    def bwd(**o):
        a = dict(ok, **o)
        return B(a["q"], a["k"], a["v"], a["a"], a["beta"], a["gate"], a["A_log"], a["cu"], a["N"], a["T"], a["H"],
                 a["dk"], a["dv"], 1.0, a["S0"], a["dout"], a["dST"], a["dq"], a["dkk"], a["dvv"], a["da"], a["db"],
                 a["dg"], a["dA"], a["dS0"], a["ws"], a["wsb"], None)

    assert bwd(dv=96) == kda.KDA_ERR_UNSUPPORTED
    assert bwd(dout=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(gate=16, dg=None) == kda.KDA_ERR_INVALID_ARG      # a gate needs its gradient
    assert bwd(wsb=10) == kda.KDA_ERR_INVALID_ARG                 # workspace too small
    assert bwd(q=8) == kda.KDA_ERR_INVALID_ARG                    # misaligned
    assert bwd(N=0, T=0) == kda.KDA_OK
    assert kda.kda_chunk_bwd_workspace_size(8192, 1, 32, 128, 128) == (8192 // 32 + 1 + 32) * 32 * 128 * 128 * 4
    # one record per (64-token chunk, head): b, W, K-, Q^ [64][d_k]; T'V then U, dU, dO [64][d_v];
    # A, X, M [64][64]; Gamma_C [d_k]; the incoming state and its gradient [d_k][d_v]
    rec = 4 * 64 * 128 + 3 * 64 * 128 + 3 * 64 * 64 + 128 + 2 * 128 * 128
    assert kda.kda_chunk_bwd_chunkwise_workspace_size(8192, 1, 32, 128, 128) == (8192 // 64 + 1) * 32 * rec * 4


def test_host_prefill_validates_on_the_host():
    import ctypes
    import torch
    cu = torch.tensor([0, 100, 260], dtype=torch.int32)
    size = kda.kda_chunk_fwd_host_buffer_size(cu, 4, 128, 128)
    assert size > 0
    assert kda.kda_chunk_fwd_host_buffer_size(cu, 4, 128, 96) == 0                 # d
    assert kda.kda_chunk_fwd_host_buffer_size(cu, 4, 128, 128, piece_tokens=32) == 0   # piece < 64
    H = lib.kda_chunk_fwd_host
    cu_p = ctypes.c_void_p(cu.data_ptr())
    alog = torch.zeros(4)
    al_p = ctypes.c_void_p(alog.data_ptr())
    bad = torch.tensor([0, 120, 100], dtype=torch.int32)                            # not monotone
    args = lambda cup, T, piece, buf, nbytes: (16, 16, 16, 16, 16, None, al_p, cup, 2, T, 4, 128, 128, 1.0, None,
                                               None, 16, 0, piece, buf, nbytes, None)
    assert H(*args(ctypes.c_void_p(bad.data_ptr()), 100, 0, 256, 1 << 40)) == kda.KDA_ERR_INVALID_ARG
    assert H(*args(cu_p, 250, 0, 256, 1 << 40)) == kda.KDA_ERR_INVALID_ARG          # cu does not end at T
    assert H(*args(cu_p, 260, 32, 256, 1 << 40)) == kda.KDA_ERR_INVALID_ARG         # piece < 64
    assert H(*args(cu_p, 260, 0, None, 0)) == kda.KDA_ERR_INVALID_ARG               # no device buffer
    assert H(*args(cu_p, 260, 0, 256, size - 1)) == kda.KDA_ERR_INVALID_ARG         # buffer too small
    assert H(*args(cu_p, 260, 0, 16, size)) == kda.KDA_ERR_INVALID_ARG              # not 256-byte aligned


def test_segment_maps_validate_on_the_host():
    fake = 256
    assert kda.lib.kda_segment_maps_workspace_size(1024, 2, 4, 96) == 0          # unsupported d
    assert kda.lib.kda_segment_maps_workspace_size(-1, 2, 4, 128) == 0
    need = kda.lib.kda_segment_maps_workspace_size(1024, 2, 4, 128)
    assert need > 0 and need % 256 == 0
    f = kda.lib.kda_segment_maps
    args = lambda **o: dict(dict(q=fake, k=fake, v=fake, a=fake, beta=fake, A_log=fake, cu=fake, N=2, T=1024, ms=512,
                                 H=4, d=128, scale=1.0, M=fake, B=fake, ws=fake, wsb=need, st=None), **o)
    call = lambda a: f(a["q"], a["k"], a["v"], a["a"], a["beta"], a["A_log"], a["cu"], a["N"], a["T"], a["ms"], a["H"],
                       a["d"], a["scale"], a["M"], a["B"], a["ws"], a["wsb"], a["st"])
    assert call(args(d=96)) == kda.KDA_ERR_UNSUPPORTED
    assert call(args(M=None)) == kda.KDA_ERR_INVALID_ARG
    assert call(args(wsb=need - 1)) == kda.KDA_ERR_INVALID_ARG
    assert call(args(ws=fake + 16)) == kda.KDA_ERR_INVALID_ARG             # workspace not 256-byte aligned
    assert call(args(q=fake + 8)) == kda.KDA_ERR_INVALID_ARG               # misaligned tensor
    assert call(args(N=0, T=0)) == kda.KDA_OK                              # nothing to do
