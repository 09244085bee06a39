"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot allocate device memory
(for example a serving engine whose device memory is all pre-reserved, or a runtime plugin whose
enqueue path must not allocate).  It runs on the library's built-in scratch array instead of a
caller workspace.  It runs the same kernel as kda_chunk_fwd on the same inputs, so its results
must equal kda_chunk_fwd's bit for bit, call after call, even though every call reuses (and leaves
behind) the same scratch contents: a scratch-reuse race or a stale record would break the equality.

This file is collected last so that a run stopping at its first failure has already run the rest.
"""
import pytest
import torch

import kda_inputs as KI

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("path", [1, 2])
def test_noalloc_matches_workspace_entry_point_on_repeated_calls(path):
    # path 1: the cluster kernel, whose chunk records live in the scratch; path 2: the per-unit
    # kernel (no scratch at all)
    import kda_chunkwise_b200 as kda
    w = KI.Workload("noalloc", (300, 77, 129, 0), 4, 128, 128, A_log="uniform",
                    init_state="normal_0.02", seed=21)
    inp = KI.make_inputs(w, "cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"])
    kda.kda_set_prefill_path(path)
    try:
        ref_out, ref_S = kda.kda_chunk_fwd(*args, gate=inp["gate"], initial_state=inp["initial_state"],
                                           out_dtype=torch.float32)
        kda.kda_sync_check()
        for call in range(2):
            out = torch.full_like(ref_out, float("nan"))
            S = torch.full_like(ref_S, float("nan"))
            kda.kda_chunk_fwd_noalloc(*args, max_seqlen=max(w.seqlens), gate=inp["gate"],
                                      initial_state=inp["initial_state"], out=out, final_state=S)
            kda.kda_sync_check()
            assert torch.equal(out, ref_out), f"call {call}: outputs differ from kda_chunk_fwd"
            assert torch.equal(S, ref_S), f"call {call}: final states differ from kda_chunk_fwd"
    finally:
        kda.kda_set_prefill_path(0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import kda_chunkwise_b200 as kda
    # With the cluster kernel, 64 sequences x 64 heads need far more chunk records than the built-in
    # 32 MiB hold; the call is rejected on the host before any pointer is touched.  (The per-unit
    # kernel, which the library picks by itself for that many units, needs no scratch.)
    fake = 256
    kda.kda_set_prefill_path(1)
    try:
        st = kda.lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, fake, 64, 64 * 512,
                                           512, 64, 128, 128, 1.0, None, None, fake, 0, None)
    finally:
        kda.kda_set_prefill_path(0)
    assert st == kda.KDA_ERR_INVALID_ARG
    msg = kda.lib.kda_last_error().decode()
    assert "scratch" in msg and "kda_chunk_fwd" in msg
    assert kda.kda_chunk_fwd_workspace_min(64 * 512, 64, 512, 64, 128, 128) == 0


def test_noalloc_runs_the_per_unit_kernel_when_cluster_records_would_not_fit():
    # 2 sequences x 28 heads = 56 units: by shape the cluster kernel (at most 66 units on B200),
    # whose records (56 x 648 KiB) exceed the 32 MiB array; with the kernel left to the shapes the
    # call runs the per-unit kernel instead, so it must equal kda_chunk_fwd on that kernel bit for bit.
    import kda_chunkwise_b200 as kda
    w = KI.Workload("noalloc56", (200, 131), 28, 128, 128, A_log="uniform", init_state="normal_0.02", seed=22)
    inp = KI.make_inputs(w, "cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"])
    assert kda.kda_prefill_path(w.num_seqs * w.H, 128, 128) == 1
    assert kda.kda_chunk_fwd_workspace_min(w.total_tokens, w.num_seqs, 200, w.H, 128, 128) > 32 << 20
    kda.kda_set_prefill_path(2)
    try:
        ref_out, ref_S = kda.kda_chunk_fwd(*args, gate=inp["gate"], initial_state=inp["initial_state"],
                                           out_dtype=torch.float32)
        kda.kda_sync_check()
    finally:
        kda.kda_set_prefill_path(0)
    out = torch.full_like(ref_out, float("nan"))
    S = torch.full_like(ref_S, float("nan"))
    kda.kda_chunk_fwd_noalloc(*args, max_seqlen=max(w.seqlens), gate=inp["gate"], initial_state=inp["initial_state"],
                              out=out, final_state=S)
    kda.kda_sync_check()
    assert torch.equal(out, ref_out) and torch.equal(S, ref_S)
