"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot allocate device memory
(for example a serving engine whose device memory is all pre-reserved, or a runtime plugin whose
enqueue path must not allocate).  It runs on the library's built-in scratch array instead of a
caller workspace, so its results must match kda_chunk_fwd's, call after call, even though every
call reuses (and leaves behind) the same scratch contents.

This file is collected last so that a run stopping at its first failure has already run the rest.
"""
import numpy as np
import pytest
import torch

import kda_inputs as KI
from parity import unit_errors, assert_unit_ok, host

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_repeated_calls():
    import kda_chunkwise_b200 as kda
    w = KI.Workload("noalloc", (300, 77, 129, 0), 4, 128, 128, A_log="uniform",
                    init_state="normal_0.02", seed=21)
    inp = KI.make_inputs(w, "cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"])
    ref_out, ref_S = kda.kda_chunk_fwd(*args, gate=inp["gate"], initial_state=inp["initial_state"],
                                       out_dtype=torch.float32)
    kda.kda_sync_check()
    cu = inp["cu_seqlens"].cpu().tolist()
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        S = torch.full_like(ref_S, float("nan"))
        kda.kda_chunk_fwd_noalloc(*args, max_seqlen=max(w.seqlens), gate=inp["gate"],
                                  initial_state=inp["initial_state"], out=out, final_state=S)
        kda.kda_sync_check()
        for n in range(w.num_seqs):
            for h in range(w.H):
                s, e = cu[n], cu[n + 1]
                err = unit_errors(host(out[s:e, h]), host(ref_out[s:e, h]), host(S[n, h]),
                                  host(ref_S[n, h]))
                assert_unit_ok(err, f"call {call}, unit ({n},{h})")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import kda_chunkwise_b200 as kda
    # 64 sequences x 64 heads of 128x128 states need far more than the built-in 32 MiB; the call
    # is rejected on the host before any pointer is touched.
    fake = 256
    st = kda.lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, fake, 64, 64 * 512,
                                       512, 64, 128, 128, 1.0, None, None, fake, 0, None)
    assert st == kda.KDA_ERR_INVALID_ARG
    msg = kda.lib.kda_last_error().decode()
    assert "scratch" in msg and "kda_chunk_fwd" in msg
