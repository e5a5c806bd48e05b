"""GPU parity at the benchmark's full sizes, in the launch configuration bench.py
times (same calls, same shapes), on sampled tokens the oracle computes one by one.

* layout: every array, exactly (the oracle layout is cheap at any size);
* dispatch: for 48 sampled tokens, every destination row's E4M3 bytes and scale
  bits (or BF16 bits) against the oracle's quantisation of that token's row;
* combine (identity experts): for the same tokens, y bit for bit against the
  oracle's fmaf chain over that token's K dequantised rows;
* combine on random expert outputs (every row different, the workload's
  weights): sampled tokens of the normal and stress batches, and every token of
  the 128-token low-latency batch, bit for bit against the oracle.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from workloads import make_custom, make_workload  # noqa: E402

from gpu_path import bf16_to_u16, torch_identity_expert  # noqa: E402


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_get_dispatch_05_b200 as m
    return m


def _run(ep, w):
    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    fp8 = w.quant == "fp8"
    x = torch.from_numpy(w.x.view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).cuda()
    wts = torch.from_numpy(w.topk_weights).cuda()
    rq = torch.empty((T * K, H), dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
    rs = torch.empty((T * K, H // 128), dtype=torch.float32, device="cuda") if fp8 else None
    ri = torch.empty(T * K, dtype=torch.int32, device="cuda")
    rw = torch.empty(T * K, dtype=torch.float32, device="cuda")
    lay = ep.Layout.empty(T, K, E, P, "cuda")
    ws = torch.empty(ep.ep_workspace_bytes(T, E, P), dtype=torch.uint8, device="cuda")
    ep.ep_workspace_init(ws)
    ep.ep_dispatch(x, idx, wts, E, P,
                   ep.EP_QUANT_FP8_E4M3_1X128 if fp8 else ep.EP_QUANT_NONE, rq, rs, ri, rw, lay, ws)
    eo = torch_identity_expert(rq, rs) if fp8 else rq
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ep.ep_combine(eo, lay, wts, y, ws)
    torch.cuda.synchronize()
    assert ep.ep_read_status(ws) == 0
    return lay, rq, rs, y


@pytest.mark.parametrize("name", ["normal", "skew", "bf16", "stress", "ll"])
def test_full_size_sampled(ep, name):
    w = make_workload(name, seed=0)
    T, H, K = w.num_tokens, w.hidden, w.num_topk
    lay, rq, rs, y = _run(ep, w)
    want = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    R = int(want["num_recv"][0])
    assert int(lay.num_recv.item()) == R
    for key in ("num_tokens_per_expert", "num_tokens_per_partition", "is_token_in_partition",
                "expert_offset", "row_of"):
        got = getattr(lay, key).cpu().numpy().reshape(want[key].shape)
        assert np.array_equal(got, want[key]), key
    assert np.array_equal(lay.src_of[:R].cpu().numpy(), want["src_of"])

    rng = np.random.default_rng(123)
    sample = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 46, replace=False)]))
    row_of = want["row_of"]
    for t in sample:
        rows = row_of[t]
        valid = rows >= 0
        if w.quant == "fp8":
            q, s = oracle.quantize_row(w.x[t])
            got_q = rq[torch.from_numpy(rows[valid]).long().cuda()].cpu().numpy()
            got_s = rs[torch.from_numpy(rows[valid]).long().cuda()].cpu().numpy()
            assert np.all(got_q == q[None, :]), t
            assert np.all(got_s.view(np.uint32) == s.view(np.uint32)[None, :]), t
            eo_t = oracle.identity_expert(q[None, :], s[None, :])
        else:
            got = bf16_to_u16(rq[torch.from_numpy(rows[valid]).long().cuda()])
            assert np.all(got == w.x[t][None, :]), t
            eo_t = w.x[t][None, :]
        # token t's K rows all hold its own (dequantised) row: reduce K copies
        eo_k = np.repeat(eo_t, K, axis=0)
        ro = np.where(valid, np.arange(K), -1).astype(np.int32)[None, :]
        y_ref, _ = oracle.combine(eo_k, ro, w.topk_weights[t][None, :])
        assert np.array_equal(bf16_to_u16(y[t:t + 1]), y_ref), t


def test_layout_many_chunks_and_rank_rounds(ep):
    # E = 4096 bounds the per-warp rank table to a few warps per round, and 30000
    # tokens fill every SM with a chunk: several rank rounds per CTA
    w = make_custom(30000, 128, 8, 4096, 64, seed=77)
    T, K = w.num_tokens, w.num_topk
    idx = torch.from_numpy(w.topk_idx).cuda()
    lay = ep.Layout.empty(T, K, 4096, 64, "cuda")
    ws = torch.empty(ep.ep_workspace_bytes(T, 4096, 64), dtype=torch.uint8, device="cuda")
    ep.ep_workspace_init(ws)
    for _ in range(2):  # the grid barrier resets itself between launches
        ep.ep_get_dispatch_layout(idx, 4096, 64, lay, ws)
        torch.cuda.synchronize()
        want = oracle.layout(w.topk_idx, 4096, 64)
        assert np.array_equal(lay.row_of.cpu().numpy(), want["row_of"])
        assert np.array_equal(lay.expert_offset.cpu().numpy(), want["expert_offset"])
        assert np.array_equal(lay.num_tokens_per_partition.cpu().numpy(),
                              want["num_tokens_per_partition"])
    assert ep.ep_read_status(ws) == 0


# ---- combine on random expert outputs, at the benchmark's launch geometry ---------

def _random_bf16(shape, seed):
    """Seeded N(0, 1) rows drawn on the device by torch (an input, like x)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


def _oracle_y(eo_rows: torch.Tensor, row_of: np.ndarray, weights: np.ndarray, tokens):
    """The oracle's combine of `tokens`, from the rows their slots name (gathered from
    the device tensor eo_rows by torch and brought to the host)."""
    ro = row_of[tokens]
    used = np.unique(ro[ro >= 0])
    rows = bf16_to_u16(eo_rows[torch.from_numpy(used).long().cuda()]) if used.size else \
        np.zeros((1, eo_rows.shape[1]), np.uint16)
    local = np.where(ro >= 0, np.searchsorted(used, np.where(ro >= 0, ro, 0)), -1).astype(np.int32)
    y, st = oracle.combine(rows, local, weights[tokens])
    assert st == 0
    return y


@pytest.mark.parametrize("name", ["normal", "stress"])
def test_full_size_combine_random_rows_sampled(ep, name):
    # every row of every token differs, so a slip in pairing a row with its weight
    # at the benchmark's geometry (persistent CTAs striding over the tokens with the
    # next token's rows prefetched) changes y
    w = make_workload(name, seed=0)
    T, H, K = w.num_tokens, w.hidden, w.num_topk
    lay, _, _, _ = _run(ep, w)
    want = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    assert np.array_equal(lay.row_of.cpu().numpy(), want["row_of"])
    R = int(want["num_recv"][0])
    eo = _random_bf16((R, H), seed=1000 + T)
    wts = torch.from_numpy(w.topk_weights).cuda()
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ep.ep_workspace_bytes(T, w.num_experts, w.num_partitions), dtype=torch.uint8,
                     device="cuda")
    ep.ep_workspace_init(ws)
    ep.ep_combine(eo, lay, wts, y, ws)
    torch.cuda.synchronize()
    assert ep.ep_read_status(ws) == 0
    rng = np.random.default_rng(7)
    sample = np.unique(np.concatenate([[0, 1, T // 2, T - 2, T - 1], rng.choice(T, 48, replace=False)]))
    y_ref = _oracle_y(eo, want["row_of"], w.topk_weights, sample)
    got = bf16_to_u16(y[torch.from_numpy(sample).long().cuda()])
    assert np.array_equal(got, y_ref)


def test_ll_full_batch_combine_random_rows(ep):
    # the whole 128-token decode batch at hidden 7168 into capacity 128 per expert,
    # every expert output row random: all of y against the oracle
    w = make_workload("ll", seed=0)
    T, H, K, E, cap = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_max_tokens
    x = torch.from_numpy(w.x.view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).cuda()
    recv_x = torch.empty((E, cap, H), dtype=torch.uint8, device="cuda")
    recv_s = torch.empty((E, cap, H // 128), dtype=torch.float32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    handle = ep.LowLatencyHandle.empty(T, K, E, cap, "cuda")
    ws = torch.empty(ep.ep_workspace_bytes(T, E, 1), dtype=torch.uint8, device="cuda")
    ep.ep_workspace_init(ws)
    ep.ep_low_latency_dispatch(x, idx, cap, E, recv_x, recv_s, cnt, handle, ws)
    eo = _random_bf16((E, cap, H), seed=2024)
    wts = torch.from_numpy(w.topk_weights).cuda()
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ep.ep_low_latency_combine(eo, handle, wts, y, ws)
    torch.cuda.synchronize()
    assert ep.ep_read_status(ws) == 0
    want = oracle.ll_dispatch(w.x, w.topk_idx, E, cap)
    assert np.array_equal(handle.row_of.cpu().numpy(), want["ll_row_of"])
    y_ref = _oracle_y(eo.view(E * cap, H), want["ll_row_of"], w.topk_weights, np.arange(T))
    assert np.array_equal(bf16_to_u16(y), y_ref)
