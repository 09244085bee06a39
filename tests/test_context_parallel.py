"""Context-parallel prefill: a sequence split into segments held by different ranks.

Over a segment the recurrence is affine in its incoming state, S -> M S + B.  CPU tests pin that
property on the oracle and run the exchange and fold of the maps over three `gloo` ranks; GPU tests
check the state-combine kernel, the maps computed by the CUDA path and the whole procedure (the
ranks emulated one after another on one GPU) against the oracle run over the unsplit sequences.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import kda_inputs as KI
import oracle
from parity import assert_unit_ok, host, unit_errors


def _unit(rng, T, d_k, d_v):
    q = rng.standard_normal((T, d_k)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, d_k)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    return dict(q=q, k=k, v=rng.standard_normal((T, d_v)), g=oracle.gate_log_decay(rng.standard_normal((T, d_k)), 0.3),
                beta=1 / (1 + np.exp(-rng.standard_normal(T))))


def _maps(u, d_k, d_v):
    _, B = oracle.recurrence_g(u["q"], u["k"], u["v"], u["g"], u["beta"], S0=np.zeros((d_k, d_v)))
    _, M = oracle.recurrence_g(u["q"], u["k"], np.zeros((len(u["q"]), d_k)), u["g"], u["beta"], S0=np.eye(d_k))
    return M, B


def test_oracle_segment_is_affine_in_its_incoming_state():
    rng = np.random.default_rng(0)
    d_k, d_v = 8, 6
    u = _unit(rng, 37, d_k, d_v)
    M, B = _maps(u, d_k, d_v)
    for _ in range(3):
        S0 = rng.standard_normal((d_k, d_v))
        _, S = oracle.recurrence_g(u["q"], u["k"], u["v"], u["g"], u["beta"], S0=S0)
        assert np.allclose(S, M @ S0 + B, atol=1e-10)


def test_oracle_folded_segment_maps_give_the_whole_sequence():
    rng = np.random.default_rng(1)
    d_k, d_v = 8, 6
    u = _unit(rng, 90, d_k, d_v)
    S0 = rng.standard_normal((d_k, d_v))
    _, S_whole = oracle.recurrence_g(u["q"], u["k"], u["v"], u["g"], u["beta"], S0=S0)
    S = S0
    for s, e in ((0, 17), (17, 64), (64, 90)):
        part = {key: val[s:e] for key, val in u.items()}
        M, B = _maps(part, d_k, d_v)
        S = M @ S + B
    assert np.allclose(S, S_whole, atol=1e-10)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cp_rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import kda_chunkwise_b200 as kda
        rng = np.random.default_rng(7)
        d_k, d_v, T = 8, 6, 60
        units = [_unit(rng, T, d_k, d_v) for _ in range(2)]   # two (sequence, head) units
        S0 = rng.standard_normal((2, d_k, d_v))
        bounds = [(0, 20), (20, 45), (45, 60)]
        s, e = bounds[rank]
        maps = [_maps({key: val[s:e] for key, val in u.items()}, d_k, d_v) for u in units]
        M = torch.tensor(np.stack([m for m, _ in maps]))
        B = torch.tensor(np.stack([b for _, b in maps]))
        S_in = kda.context_parallel_states(M, B, torch.tensor(S0),
                                           combine=lambda m, s_, b: torch.matmul(m, s_) + b)
        expect = []
        for i, u in enumerate(units):   # the oracle's state at the start of this rank's segment
            head = {key: val[:s] for key, val in u.items()}
            expect.append(S0[i] if s == 0 else oracle.recurrence_g(head["q"], head["k"], head["v"], head["g"],
                                                                    head["beta"], S0=S0[i])[1])
        np.savez(os.path.join(out_dir, f"cp{rank}.npz"), got=S_in.numpy(), expect=np.stack(expect))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_three_gloo_ranks_fold_the_maps_in_order(tmp_path):
    world = 3
    mp.spawn(_cp_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        z = np.load(tmp_path / f"cp{r}.npz")
        assert np.allclose(z["got"], z["expect"], atol=1e-10), f"rank {r}"


# ---- GPU ------------------------------------------------------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_state_combine_kernel(dk, dv):
    import kda_chunkwise_b200 as kda
    g = torch.Generator(device="cuda").manual_seed(dk + dv)
    M = torch.randn((3, 5, dk, dk), generator=g, device="cuda") / dk ** 0.5
    S = torch.randn((3, 5, dk, dv), generator=g, device="cuda")
    B = torch.randn((3, 5, dk, dv), generator=g, device="cuda")
    out = kda.kda_state_combine(M, S, B)
    kda.kda_sync_check()
    ref = host(M) @ host(S) + host(B)
    assert np.abs(host(out) - ref).max() <= 1e-4 * np.abs(ref).max()
    with pytest.raises(kda.KDAError):
        kda.kda_state_combine(M, S, B, out=S)   # S_out may not alias S_in


def _split(inp, cu, seg_bounds):
    """Segment r of every sequence, packed: per-rank inputs and cu_seqlens."""
    parts = []
    for r in range(len(seg_bounds[0])):
        rows, cu_r = [], [0]
        for n in range(len(cu) - 1):
            s, e = seg_bounds[n][r]
            rows.append(torch.arange(cu[n] + s, cu[n] + e))
            cu_r.append(cu_r[-1] + e - s)
        idx = torch.cat(rows).to("cuda")
        part = {key: inp[key].index_select(0, idx).contiguous() for key in ("q", "k", "v", "a", "beta", "gate")}
        part["cu_seqlens"] = torch.tensor(cu_r, dtype=torch.int32, device="cuda")
        part["idx"] = idx
        parts.append(part)
    return parts


@pytest.mark.gpu
def test_context_parallel_prefill_matches_the_unsplit_oracle():
    import kda_chunkwise_b200 as kda
    from parity import check_units
    w = KI.Workload("cp", (300, 190), 2, 128, 128, init_state="normal_0.02", seed=21)
    inp = KI.make_inputs(w, "cuda")
    cu = inp["cu_seqlens"].cpu().tolist()
    # three segments per sequence (uneven, not multiples of the chunk)
    seg_bounds = [[(0, 70), (70, 200), (200, 300)], [(0, 64), (64, 100), (100, 190)]]
    parts = _split(inp, cu, seg_bounds)
    maps = [kda.kda_segment_maps(p["q"], p["k"], p["v"], p["a"], p["beta"], inp["A_log"], p["cu_seqlens"])
            for p in parts]
    out = torch.empty((w.total_tokens, w.H, w.d_v), dtype=torch.float32, device="cuda")
    S = inp["initial_state"].clone()
    for r, p in enumerate(parts):   # rank r's fold of ranks 0..r-1, then its corrected pass
        if r > 0:
            S = kda.kda_state_combine(maps[r - 1][0], S_prev, maps[r - 1][1])
        o, S_out = kda.kda_chunk_fwd(p["q"], p["k"], p["v"], p["a"], p["beta"], inp["A_log"], p["cu_seqlens"],
                                     gate=p["gate"], initial_state=S, out_dtype=torch.float32)
        out.index_copy_(0, p["idx"], o)
        S_prev = S
    kda.kda_sync_check()
    check_units(inp, out, S_out, [(n, h) for n in range(w.num_seqs) for h in range(w.H)])


def _cp_gpu_rank(rank, world, port, out_dir):
    """Rank `rank` of a gloo group whose ranks share one GPU: it holds segment `rank` of every
    sequence and calls kda_context_parallel_fwd itself (the maps are exchanged over gloo through
    host copies; no rank's kernel waits on another's)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import kda_chunkwise_b200 as kda
        w = KI.Workload("cp_api", (300, 190), 2, 128, 128, A_log="uniform", init_state="normal_0.02", seed=22)
        inp = KI.make_inputs(w, "cuda")
        cu = inp["cu_seqlens"].cpu().tolist()
        seg_bounds = [[(0, 70), (70, 200), (200, 300)], [(0, 64), (64, 100), (100, 190)]]
        p = _split(inp, cu, seg_bounds)[rank]
        out, S = kda.kda_context_parallel_fwd(p["q"], p["k"], p["v"], p["a"], p["beta"], inp["A_log"], p["cu_seqlens"],
                                              gate=p["gate"], initial_state=inp["initial_state"],
                                              out_dtype=torch.float32)
        kda.kda_sync_check()
        np.savez(os.path.join(out_dir, f"cpgpu{rank}.npz"), out=out.cpu().numpy(), S=S.cpu().numpy(),
                 idx=p["idx"].cpu().numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_context_parallel_entry_point_over_three_ranks_matches_the_unsplit_oracle(tmp_path):
    """kda_context_parallel_fwd as shipped (segment maps, all-gather, kda_state_combine fold,
    corrected pass) on three ranks, against the oracle run over the unsplit sequences: the
    outputs of every segment and, from the last rank, the final states."""
    from parity import check_units
    world = 3
    mp.spawn(_cp_gpu_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    w = KI.Workload("cp_api", (300, 190), 2, 128, 128, A_log="uniform", init_state="normal_0.02", seed=22)
    inp = KI.make_inputs(w, "cuda")
    out = torch.empty((w.total_tokens, w.H, w.d_v), dtype=torch.float32)
    for r in range(world):
        z = np.load(tmp_path / f"cpgpu{r}.npz")
        out[torch.from_numpy(z["idx"])] = torch.from_numpy(z["out"])
    S_last = torch.from_numpy(np.load(tmp_path / f"cpgpu{world - 1}.npz")["S"])
    check_units(inp, out, S_last, [(n, h) for n in range(w.num_seqs) for h in range(w.H)])


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("a_mean", [0.0, -8.0])
def test_one_pass_segment_maps_match_the_oracle_and_the_two_pass_maps(d, a_mean):
    # kda_segment_maps in one pass ([0 | v] from [I | 0]) against the oracle's maps of each unit
    # (B from S = 0, M from S = I with v = 0) and against the two-call form, on ragged sequences.
    # With fading decays (a ~ N(0, 1)) M shrinks towards zero (as e^{b}), so errors are also bounded
    # against the scale of the identity (1e-4 sqrt(d)); with almost no fade (a ~ N(-8, 1)) M stays
    # of the identity's size.
    import kda_chunkwise_b200 as kda
    w = KI.Workload("maps", (300, 77, 129), 2, d, d, A_log="uniform", a_mean=a_mean, seed=23)
    inp = KI.make_inputs(w, "cuda")
    M1, B1 = kda.kda_segment_maps(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"])
    M2, B2 = kda.kda_segment_maps(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                                  single_pass=False)
    kda.kda_sync_check()
    floor = 1e-4 * d ** 0.5
    for x, y in ((M1, M2), (B1, B2)):
        assert float((x - y).norm()) <= 2e-3 * float(y.norm()) + floor
    cu = inp["cu_seqlens"].cpu().tolist()
    A_log = host(inp["A_log"])
    for n in range(w.num_seqs):
        s, e = cu[n], cu[n + 1]
        for h in range(w.H):
            q, k, v = (host(inp[x][s:e, h]) for x in ("q", "k", "v"))
            g = oracle.gate_log_decay(host(inp["a"][s:e, h]), float(A_log[h]))
            beta = host(inp["beta"][s:e, h])
            _, B_ref = oracle.recurrence_g(q, k, v, g, beta, S0=np.zeros((d, d)))
            _, M_ref = oracle.recurrence_g(q, k, np.zeros((e - s, d)), g, beta, S0=np.eye(d))
            for got, ref, name in ((host(M1[n, h]), M_ref, "M"), (host(B1[n, h]), B_ref, "B")):
                err = np.linalg.norm(got - ref)
                assert err <= 5e-3 * np.linalg.norm(ref) + floor, f"unit ({n},{h}) {name}: |err| {err:.2e}"
