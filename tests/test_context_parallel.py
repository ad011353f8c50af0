"""KDA context parallelism: a batch of sequences split along T over ranks, only the fixed-size
state maps exchanged, each rank's outputs corrected once its incoming state is known.

CPU: the orchestration with an fp64 stand-in for the per-segment kernels (the oracle), both
as ranks emulated in one process and as real gloo ranks (world sizes 2 and 3, ragged
segments); the C ABI's checks of the composition entry point.
GPU: the same steps on the library's kernels, ranks emulated one after another on one device
(no rank waits for another inside a kernel), against the oracle on the whole sequence; the
composition kernel against a CPU matmul.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS
from linear_attention_recurrence_forward_b200 import context_parallel as cp
from helpers import max_rel_err, random_problem


class OracleOps:
    """fp64 CPU stand-in for the kernels (tests only)."""

    state_dtype = torch.float64

    def forward(self, q, k, v, g, beta, S0):
        o, ST = oracle.forward(q, k, v, g, beta, None if S0 is None else S0)
        return torch.from_numpy(o), torch.from_numpy(ST)

    def compose(self, M, S, N):
        return torch.matmul(M, S) + N

    def correct(self, C, S, o0):
        return o0 + torch.einsum("bthi,bhij->bthj", C, S)


def split_points(T, world, seed):
    rng = np.random.default_rng(seed)
    cuts = sorted(rng.choice(np.arange(1, T), size=world - 1, replace=False).tolist())
    return [0] + cuts + [T]


def problem(B=2, T=150, H=2, dk=8, dv=6, seed=0):
    """Slow decay (g in [-0.05, 0)), so each segment's map carries the state it is given."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = random_problem(rng, B, T, H, dk, dv, g_lo=-0.05)
    return [torch.from_numpy(x) for x in (q, k, v, g, beta)], torch.from_numpy(S0)


def emulate(xs, S0, bounds, ops):
    world = len(bounds) - 1
    segs = [[x[:, bounds[r]:bounds[r + 1]].contiguous() for x in xs] for r in range(world)]
    first = [cp.rank_first_step(r, world, *segs[r], S0=S0, ops=ops) for r in range(world)]
    Ms = [f[0] for f in first]
    Ns = [f[1] for f in first]
    outs, S_end = [first[0][2]], first[0][3]
    for r in range(1, world):
        S_in = cp.incoming_state(Ms, Ns, r, ops)
        M, N, o0, _, C = first[r]
        o, S_end = cp.rank_finish(S_in, o0, C, M, N, ops=ops)
        outs.append(o)
    return torch.cat(outs, dim=1), S_end


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_emulated_ranks_match_the_whole_sequence(world):
    xs, S0 = problem(seed=world)
    bounds = split_points(xs[0].shape[1], world, seed=world)
    o, ST = emulate(xs, S0, bounds, OracleOps())
    o_ref, ST_ref = oracle.forward(*xs, S0)
    assert max_rel_err(o.numpy(), o_ref) < 1e-12 and max_rel_err(ST.numpy(), ST_ref) < 1e-12


def test_segment_map_is_the_affine_map():
    xs, S0 = problem(T=40, seed=7)
    M, N = cp.segment_map(*xs, ops=OracleOps())
    assert float(M.abs().max()) > 0.1   # the map is far from zero at this decay
    _, ST = oracle.forward(*xs, S0)
    assert max_rel_err((torch.matmul(M, S0) + N).numpy(), ST) < 1e-12
    # plausible slips do not pass: the transposed map, or dropping N
    assert max_rel_err((torch.matmul(M.transpose(-1, -2), S0) + N).numpy(), ST) > 1e-3
    assert max_rel_err(torch.matmul(M, S0).numpy(), ST) > 1e-3


def test_correction_operand_is_the_state_map_read_out():
    """C_t from the v = 0, S0 = I run satisfies o_t = o0_t + S^T C_t for any start state S, token by
    token, and its final state is the map M (fp64 stand-in)."""
    xs, S0 = problem(T=70, seed=9)
    o0, N, C, M = cp.segment_pass(*xs, ops=OracleOps())
    o_ref, ST_ref = oracle.forward(*xs, S0)
    o = o0 + torch.einsum("bthi,bhij->bthj", C, S0)
    assert max_rel_err(o.numpy(), o_ref) < 1e-12
    assert max_rel_err((torch.matmul(M, S0) + N).numpy(), ST_ref) < 1e-12
    # plausible slips do not pass: the correction dropped, or the segment's final map used for every
    # token instead of the map up to that token
    assert max_rel_err(o0.numpy(), o_ref) > 1e-3
    q = xs[0]
    o_end = o0 + torch.einsum("bthi,bhij->bthj", q, torch.matmul(M, S0))
    assert max_rel_err(o_end.numpy(), o_ref) > 1e-3


def _rank_main(rank, world, port, bounds, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        xs, S0 = problem(seed=11)
        seg = [x[:, bounds[rank]:bounds[rank + 1]].contiguous() for x in xs]
        o, final = cp.context_parallel_forward(*seg, S0=S0, ops=OracleOps())
        out[rank] = (o.numpy(), final.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_the_whole_sequence(world):
    xs, S0 = problem(seed=11)
    bounds = split_points(xs[0].shape[1], world, seed=world + 20)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = 29600 + (os.getpid() % 500) + 7 * world
    mp.start_processes(_rank_main, args=(world, port, bounds, out), nprocs=world, join=True, start_method="spawn")
    o = np.concatenate([out[r][0] for r in range(world)], axis=1)
    o_ref, ST_ref = oracle.forward(*xs, S0)
    assert max_rel_err(o, o_ref) < 1e-12
    for r in range(world):
        assert max_rel_err(out[r][1], ST_ref) < 1e-12


# ---------------------------------------------------------------------- C ABI checks (CPU)

BASE = 0x7F0000000000
SZ = 1 << 30
OK, INVALID, UNSUPPORTED, MISALIGNED = (STATUS[n] for n in
                                        ("KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                         "KDA_ERR_MISALIGNED"))


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrence_forward_b200 import build
    build.build()
    return kda.lib()


def test_compose_rejects_bad_arguments(L):
    M, S, N, O = (BASE + i * SZ for i in range(4))
    assert L.kda_state_compose(M, S, N, O, 0, 128, 128, None) == INVALID
    assert L.kda_state_compose(M, S, N, O, 4, 96, 128, None) == UNSUPPORTED
    assert L.kda_state_compose(None, S, N, O, 4, 128, 128, None) == INVALID
    assert L.kda_state_compose(M, S, N, None, 4, 128, 128, None) == INVALID
    assert L.kda_state_compose(M + 8, S, N, O, 4, 128, 128, None) == MISALIGNED
    assert L.kda_state_compose(M, S, N, M + 4096, 4, 128, 128, None) == INVALID     # out inside M
    assert L.kda_state_compose(M, S, N, S + 4096, 4, 128, 128, None) == INVALID     # partial overlap with S
    assert L.kda_state_compose(M, S, N, N - 4096, 4, 128, 128, None) == INVALID     # partial overlap with N


# ---------------------------------------------------------------------- GPU

@pytest.mark.gpu
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_compose_kernel_matches_a_cpu_matmul(dk, dv):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(dk + dv)
    M = torch.randn((3, 5, dk, dk), generator=gen, device="cuda") * 0.1
    S = torch.randn((3, 5, dk, dv), generator=gen, device="cuda")
    N = torch.randn((3, 5, dk, dv), generator=gen, device="cuda")
    ref = (M.double().cpu() @ S.double().cpu() + N.double().cpu()).numpy()
    out = kda.kda_state_compose(M, S, N)
    assert max_rel_err(out.double().cpu().numpy(), ref) < 1e-5
    # in place over S and over N
    S2 = S.clone()
    kda.kda_state_compose(M, S2, N, out=S2)
    N2 = N.clone()
    kda.kda_state_compose(M, S, N2, out=N2)
    torch.cuda.synchronize()
    assert torch.equal(S2, out) and torch.equal(N2, out)
    # N omitted is zero
    ref0 = (M.double().cpu() @ S.double().cpu()).numpy()
    assert max_rel_err(kda.kda_state_compose(M, S).double().cpu().numpy(), ref0) < 1e-5


def test_output_correct_rejects_bad_arguments(L):
    C, S, Oi, Oo = (BASE + i * SZ for i in range(4))
    f = L.kda_output_correct
    assert f(C, S, Oi, Oo, 0, 64, 2, 128, 128, 0, None) == INVALID
    assert f(C, S, Oi, Oo, 1, -1, 2, 128, 128, 0, None) == INVALID
    assert f(C, S, Oi, Oo, 1, 64, 2, 96, 128, 0, None) == UNSUPPORTED
    assert f(C, S, Oi, Oo, 1, 64, 2, 128, 128, 5, None) == UNSUPPORTED
    assert f(None, S, Oi, Oo, 1, 64, 2, 128, 128, 0, None) == INVALID
    assert f(C + 8, S, Oi, Oo, 1, 64, 2, 128, 128, 0, None) == MISALIGNED
    assert f(C, S, Oi, C + 4096, 1, 64, 2, 128, 128, 0, None) == INVALID    # out inside C
    assert f(C, S, Oi, Oi + 4096, 1, 64, 2, 128, 128, 0, None) == INVALID   # out partly over o_in
    assert f(C, S, Oi, Oo, 1, 0, 2, 128, 128, 0, None) == OK                # no tokens: nothing to do


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,dk,dv,T", [("bf16", 128, 128, 300), ("bf16", 128, 128, 128), ("bf16", 128, 128, 1),
                                           # 16, 17 and 40 tiles of 128 tokens: one run of tiles per CTA, a
                                           # second CTA with one tile, three CTAs with a ragged last tile
                                           ("bf16", 128, 128, 2048), ("bf16", 128, 128, 2049), ("bf16", 128, 128, 5000),
                                           ("bf16", 64, 128, 77), ("fp32", 64, 64, 100), ("fp32", 128, 128, 33)])
def test_output_correct_kernel_matches_a_cpu_product(dtype, dk, dv, T):
    from linear_attention_recurrence_forward_b200.inputs import torch_dtype
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T + dk)
    dt = torch_dtype(dtype)
    C = (torch.randn((2, T, 3, dk), generator=gen, device="cuda") * 0.3).to(dt)
    o0 = torch.randn((2, T, 3, dv), generator=gen, device="cuda").to(dt)
    S = torch.randn((2, 3, dk, dv), generator=gen, device="cuda") * 0.2
    ref = (o0.double().cpu() + torch.einsum("bthi,bhij->bthj", C.double().cpu(), S.double().cpu())).numpy()
    out = kda.kda_output_correct(C, S, o0)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    tol = 2e-2 if dtype == "bf16" else 1e-5
    assert max_rel_err(out.double().cpu().numpy(), ref) < tol
    # in place over o_in
    o1 = o0.clone()
    kda.kda_output_correct(C, S, o1, out=o1)
    torch.cuda.synchronize()
    assert torch.equal(o1, out)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,world,T,zg_mean", [("bf16", 2, 1000, -8.0), ("bf16", 4, 2100, -8.0),
                                                   ("bf16", 3, 2000, 0.0), ("fp32", 3, 400, -8.0)])
def test_context_parallel_steps_on_one_gpu(dtype, world, T, zg_mean):
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    d = 128 if dtype == "bf16" else 64
    # slow decay (z ~ N(-8, 1), g ~ -2e-3), so the composed states matter; and the recipe's decay
    # (z ~ N(0, 1)), under which the maps M are far from the identity
    q, k, v, g, beta, S0 = make_prefill_inputs(2, T, 3, d, d, dtype, seed=5, s0_std=0.05, zg_mean=zg_mean,
                                               device="cuda")
    bounds = [0] + [(T * r) // world // 64 * 64 + 17 * r for r in range(1, world)] + [T]
    o, ST = emulate([q, k, v, g, beta], S0, bounds, cp.CudaOps())
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0)
    tol = 2e-2 if dtype == "bf16" else 1e-4
    eo = max_rel_err(o.double().cpu().numpy(), o_ref)
    es = max_rel_err(ST.double().cpu().numpy(), ST_ref)
    assert eo <= tol and es <= tol, (eo, es)


def _nccl_rank_main(rank, world, port, out):
    """One rank of the NCCL path on its own GPU (context_parallel_forward with the CUDA kernels)."""
    from datetime import timedelta
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", rank))
    try:
        q, k, v, g, beta, S0 = make_prefill_inputs(2, 500, 3, 128, 128, "bf16", seed=21, s0_std=0.05, device="cuda")
        o, final = cp.context_parallel_forward(q, k, v, g, beta, S0=S0)
        o_ref, ST_ref = kda.kda_forward_chunked(q, k, v, g, beta, S0)
        torch.cuda.synchronize()
        out[rank] = (bool(torch.equal(o, o_ref)), bool(torch.equal(final, ST_ref)))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_nccl_path_on_one_gpu():
    """context_parallel_forward over a one-rank NCCL group: the collectives run on device tensors and the
    result equals the plain prefill bitwise (rank 0 runs its segment for real).  The exchange between
    several GPUs is covered by the gloo ranks and the emulated GPU ranks above; one GPU is all a run has."""
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = 29950 + (os.getpid() % 40)
    mp.start_processes(_nccl_rank_main, args=(1, port, out), nprocs=1, join=True, start_method="spawn")
    assert out[0] == (True, True)
