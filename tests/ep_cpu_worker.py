"""One rank of the CPU test of EpGroup's exchange (spawned by tests/test_ep_cpu.py).

The one-GPU kernels are replaced by CPU stand-ins built from the oracle, so that
what runs is the exchange itself: row counts, all_to_all splits, per-expert
counts and the return path, over gloo between real processes."""
import datetime
import os
import sys

import numpy as np


def _stand_ins(oracle, torch):
    def dispatch(x, idx, w, E, P, quant, q, s, ri, rw, lay, ws, stream=None):
        xs = x.view(torch.int16).numpy().view(np.uint16)
        d = oracle.dispatch(xs, idx.numpy(), w.numpy(), E, P, quant="fp8" if quant else "none")
        R = int(d["num_recv"][0])
        if quant:
            q[:R] = torch.from_numpy(d["recv_x"])
            s[:R] = torch.from_numpy(d["recv_scales"])
        else:
            q[:R] = torch.from_numpy(d["recv_x"].view(np.int16)).view(torch.bfloat16)
        ri[:R] = torch.from_numpy(d["recv_topk_idx"])
        rw[:R] = torch.from_numpy(d["recv_topk_weights"])
        for name in ("num_tokens_per_expert", "num_tokens_per_partition",
                     "is_token_in_partition", "expert_offset", "row_of", "num_recv"):
            getattr(lay, name).copy_(torch.from_numpy(np.ascontiguousarray(d[name])).view(
                getattr(lay, name).shape))
        lay.src_of[:R] = torch.from_numpy(d["src_of"])

    def combine(eo, lay, w, y, ws, stream=None):
        bits = eo.view(torch.int16).numpy().view(np.uint16)
        yb, _ = oracle.combine(bits, lay.row_of.numpy(), w.numpy())
        y.copy_(torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16))

    return dispatch, combine


def run(rank: int, world: int, port: int, out_dir: str) -> None:
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    status = "failed"
    try:
        import oracle
        from combine_get_dispatch_05_b200 import ep_group
        from workloads import make_custom

        stand_dispatch, stand_combine = _stand_ins(oracle, torch)
        ep_group._lib.ep_dispatch = stand_dispatch
        ep_group._lib.ep_combine = stand_combine
        ep_group._lib.ep_workspace_init = lambda ws, stream=None: None

        E, H, K = 48, 256, 5
        tokens = [0 if r == world - 1 and world > 2 else 90 + 37 * r for r in range(world)]
        loads = [make_custom(tokens[r], H, K, E, world, seed=200 + r, mask_frac=0.1)
                 for r in range(world)]
        w = loads[rank]
        g = ep_group.EpGroup(E, device="cpu")
        x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16)
        idx = torch.from_numpy(w.topk_idx)
        wts = torch.from_numpy(w.topk_weights)
        epp = E // world
        for quant in ("fp8", "none"):
            recv_x, ri, rw, per_expert, ctx = g.dispatch(x, idx, wts, use_fp8=quant == "fp8")
            want_x, want_i, want_w, want_cnt = [], [], [], []
            for ws in loads:
                d = oracle.dispatch(ws.x, ws.topk_idx, ws.topk_weights, E, world, quant=quant)
                lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
                want_x.append(d["recv_x"][lo:hi])
                want_i.append(d["recv_topk_idx"][lo:hi])
                want_w.append(d["recv_topk_weights"][lo:hi])
                want_cnt.append(d["num_tokens_per_expert"][rank * epp:(rank + 1) * epp])
            # identity experts: the received rows, dequantised as the oracle does
            if quant == "fp8":
                got_x = recv_x[0].view(torch.uint8).numpy()
                eo_bits = oracle.identity_expert(got_x, recv_x[1].numpy())
            else:
                got_x = recv_x.view(torch.int16).numpy().view(np.uint16)
                eo_bits = oracle.identity_expert(got_x, None, quant="none")
            assert np.array_equal(got_x, np.concatenate(want_x)), quant
            assert np.array_equal(ri.numpy(), np.concatenate(want_i)), quant
            assert np.array_equal(rw.numpy().view(np.uint32),
                                  np.concatenate(want_w).view(np.uint32)), quant
            assert np.array_equal(per_expert.numpy(), np.stack(want_cnt)), quant
            eo = torch.from_numpy(np.ascontiguousarray(eo_bits).view(np.int16)).view(torch.bfloat16)
            y = g.combine(eo, ctx, wts)
            mine = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, world, quant=quant)
            eo_mine = oracle.identity_expert(mine["recv_x"], mine.get("recv_scales"), quant=quant)
            y_ref, _ = oracle.combine(eo_mine, mine["row_of"], w.topk_weights)
            assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16), y_ref), quant
        status = "ok"
    finally:
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(status)
        dist.destroy_process_group()
