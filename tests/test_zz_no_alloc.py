"""ep_get_dispatch_layout_static: the layout for callers that cannot allocate
device memory (an engine that owns all of HBM through its own pool, a plugin
that must not allocate while enqueueing, a latency-critical path that cannot
afford cudaMalloc's implicit synchronisation).  It keeps its scratch in a fixed
array inside the library instead of a caller-provided workspace.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  It also passes when run alone.
"""
import ctypes

import pytest

from workloads import make_custom, make_workload


@pytest.fixture(scope="module")
def ep():
    import __graft_entry__

    __graft_entry__.build()
    import combine_get_dispatch_05_b200 as m

    return m


def test_static_layout_rejects_batches_beyond_its_scratch(ep):
    # needs no GPU: the size check runs before anything touches CUDA
    limit = 1 << 20
    f = 0x100000
    lay = ep._lib.ep_layout(f, f, f, f, f, f, f)
    T = 300_000
    assert ep.ep_workspace_bytes(T, 256, 8) > limit
    st = ep.lib.ep_get_dispatch_layout_static(T, 8, 256, 8, f, ctypes.byref(lay), None)
    assert st == ep.EP_ERR_WORKSPACE


@pytest.mark.gpu
def test_static_layout_matches_workspace_layout_twice(ep):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    stream = torch.cuda.current_stream()
    # calls in a row with different batches: none may see an earlier call's
    # leftovers in the shared scratch.  The first and third take the multi-CTA
    # layout (per-chunk counts and the grid-barrier word live in the scratch; the
    # third has fewer tokens and other E / P than the first), the second the
    # one-CTA layout (header only).
    batches = [make_workload("normal", seed=31, num_tokens=1000, hidden=128),
               make_custom(300, 128, 6, 64, 16, seed=32, mask_frac=0.1),
               make_custom(700, 128, 6, 64, 16, seed=33, mask_frac=0.1)]
    for w in batches:
        T, K, E, P = w.num_tokens, w.num_topk, w.num_experts, w.num_partitions
        idx = torch.from_numpy(w.topk_idx).cuda()
        ref = ep.Layout.empty(T, K, E, P, "cuda")
        ws = torch.empty(ep.ep_workspace_bytes(T, E, P), dtype=torch.uint8, device="cuda")
        ep.ep_workspace_init(ws)
        ep.ep_get_dispatch_layout(idx, E, P, ref, ws)
        got = ep.Layout.empty(T, K, E, P, "cuda")
        c = got.c()
        st = ep.lib.ep_get_dispatch_layout_static(T, K, E, P, idx.data_ptr(), ctypes.byref(c),
                                                  stream.cuda_stream)
        assert st == ep.EP_OK
        torch.cuda.synchronize()
        R = int(ref.num_recv.item())
        assert int(got.num_recv.item()) == R
        for name in ("num_tokens_per_expert", "num_tokens_per_partition",
                     "is_token_in_partition", "expert_offset", "row_of"):
            assert torch.equal(getattr(got, name), getattr(ref, name)), name
        assert torch.equal(got.src_of[:R], ref.src_of[:R])
