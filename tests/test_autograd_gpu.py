"""chunk_kda, the prefill as a torch.autograd function: the gradients autograd delivers are those of
kda_chunk_bwd called directly with the same upstream gradients (itself checked against the oracle's
reverse-mode derivative in test_backward_gpu.py), cast to each input's dtype."""
import pytest
import torch

import kda_inputs as KI

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    return m


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_autograd_gradients_are_the_backward_kernels(kda, out_dtype):
    w = KI.Workload("ag", (90, 0, 41), 2, 128, 128, A_log="uniform", init_state="normal_0.02", seed=51)
    inp = KI.make_inputs(w, "cuda")
    names = ("q", "k", "v", "a", "beta", "A_log", "gate", "initial_state")
    leaf = {n: inp[n].clone().requires_grad_(True) for n in names}
    g_ = torch.Generator(device="cuda").manual_seed(52)
    W1 = torch.randn((w.total_tokens, w.H, w.d_v), generator=g_, device="cuda")
    W2 = torch.randn((w.num_seqs, w.H, w.d_k, w.d_v), generator=g_, device="cuda")
    out, S = kda.chunk_kda(leaf["q"], leaf["k"], leaf["v"], leaf["a"], leaf["beta"], leaf["A_log"],
                           inp["cu_seqlens"], gate=leaf["gate"], initial_state=leaf["initial_state"],
                           scale=0.8, out_dtype=out_dtype)
    ((out.float() * W1).sum() + (S * W2).sum()).backward()
    dout = W1.to(out_dtype).float()   # the gradient reaching a bf16 output is rounded to bf16
    ref = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                            dout, gate=inp["gate"], initial_state=inp["initial_state"], dfinal_state=W2, scale=0.8)
    kda.kda_sync_check()
    pairs = {"q": "dq", "k": "dk", "v": "dv", "a": "da", "beta": "dbeta", "gate": "dgate",
             "initial_state": "dinitial_state"}
    for n, key in pairs.items():
        assert leaf[n].grad is not None and leaf[n].grad.dtype == inp[n].dtype, n
        assert torch.equal(leaf[n].grad, ref[key].to(inp[n].dtype)), n
    # dA_log is summed with atomics over sequences and column slices: equal up to the order
    assert torch.allclose(leaf["A_log"].grad, ref["dA_log"], rtol=1e-5, atol=1e-6)
