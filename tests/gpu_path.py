"""Helpers for the GPU tests: run the CUDA path through the C ABI (via the thin
binding) on host inputs and bring every output back as numpy arrays.

Buffers are allocated with a tail canary (bytes 0xA5) and the receive buffers
are pre-filled with a sentinel, so the tests can check that kernels write
nothing outside the rows they own.
"""
from __future__ import annotations

import numpy as np
import torch

CANARY = 0xA5
CANARY_BYTES = 4096


def dev_u16_as_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).cuda().view(
        torch.bfloat16)


def bf16_to_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Guarded:
    """A device tensor followed by a canary tail of CANARY_BYTES bytes."""

    def __init__(self, shape, dtype, fill_byte=CANARY):
        n = int(np.prod(shape)) if len(shape) else 1
        itemsize = torch.empty(0, dtype=dtype).element_size()
        nbytes = n * itemsize
        self.raw = torch.full((nbytes + CANARY_BYTES,), fill_byte, dtype=torch.uint8, device="cuda")
        self.t = self.raw[:nbytes].view(dtype).view(*shape) if n else torch.empty(
            shape, dtype=dtype, device="cuda")
        self.nbytes = nbytes

    def canary_ok(self) -> bool:
        return bool((self.raw[self.nbytes:] == CANARY).all().item())


def gpu_layout(ep, topk_idx: np.ndarray, E: int, P: int, workspace=None):
    T, K = topk_idx.shape
    idx = torch.from_numpy(np.ascontiguousarray(topk_idx, np.int64)).cuda()
    lay = ep.Layout.empty(T, K, E, P, "cuda")
    ws = workspace if workspace is not None else new_workspace(ep, T, E, P)
    ep.ep_get_dispatch_layout(idx, E, P, lay, ws)
    torch.cuda.synchronize()
    return lay, ws


def new_workspace(ep, T, E, P):
    ws = torch.empty(ep.ep_workspace_bytes(max(T, 1), E, P), dtype=torch.uint8, device="cuda")
    ep.ep_workspace_init(ws)
    return ws


def layout_numpy(lay, T, K):
    R = int(lay.num_recv.item())
    return dict(
        num_tokens_per_expert=lay.num_tokens_per_expert.cpu().numpy(),
        num_tokens_per_partition=lay.num_tokens_per_partition.cpu().numpy(),
        is_token_in_partition=lay.is_token_in_partition.cpu().numpy(),
        expert_offset=lay.expert_offset.cpu().numpy(),
        row_of=lay.row_of.cpu().numpy().reshape(T, K),
        src_of=lay.src_of.cpu().numpy()[:R],
        num_recv=np.array([R], np.int32),
    )


def quant_code(ep, quant: str) -> int:
    return {"none": ep.EP_QUANT_NONE, "fp8": ep.EP_QUANT_FP8_E4M3_1X128,
            "fp8_pow2": ep.EP_QUANT_FP8_E4M3_1X128_POW2}[quant]


def gpu_dispatch(ep, w, workspace=None, quant=None):
    """Layout + dispatch of workload `w` on the GPU; returns (numpy dict, device state)."""
    quant = w.quant if quant is None else quant
    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    fp8 = quant in ("fp8", "fp8_pow2")
    x = dev_u16_as_bf16(w.x)
    idx = torch.from_numpy(np.ascontiguousarray(w.topk_idx)).cuda()
    wts = torch.from_numpy(np.ascontiguousarray(w.topk_weights)).cuda()
    rows = max(T * K, 1)
    recv_x = Guarded((rows, H), torch.uint8 if fp8 else torch.bfloat16)
    recv_s = Guarded((rows, max(H // 128, 1)), torch.float32) if fp8 else None
    recv_i = Guarded((rows,), torch.int32)
    recv_w = Guarded((rows,), torch.float32)
    lay = ep.Layout.empty(T, K, E, P, "cuda")
    ws = workspace if workspace is not None else new_workspace(ep, T, E, P)
    ep.ep_dispatch(x, idx, wts, E, P, quant_code(ep, quant),
                   recv_x.t, recv_s.t if fp8 else None, recv_i.t, recv_w.t, lay, ws)
    torch.cuda.synchronize()
    out = layout_numpy(lay, T, K)
    R = int(out["num_recv"][0])
    if fp8:
        out["recv_x"] = recv_x.t[:R].cpu().numpy()
        out["recv_scales"] = recv_s.t[:R, : H // 128].cpu().numpy()
    else:
        out["recv_x"] = bf16_to_u16(recv_x.t[:R])
    out["recv_topk_idx"] = recv_i.t[:R].cpu().numpy()
    out["recv_topk_weights"] = recv_w.t[:R].cpu().numpy()
    # rows >= R were never written (still the 0xA5 fill) and the tails are intact
    untouched = bool((recv_x.raw[R * H * (1 if fp8 else 2):] == 0xA5).all().item())
    guards = [recv_x, recv_i, recv_w] + ([recv_s] if fp8 else [])
    out["canaries_ok"] = all(g.canary_ok() for g in guards) and untouched
    state = dict(x=x, idx=idx, wts=wts, recv_x=recv_x.t, recv_s=recv_s.t if fp8 else None,
                 layout=lay, ws=ws)
    return out, state


def gpu_combine(ep, expert_out_u16: np.ndarray, lay, topk_weights: np.ndarray, ws):
    T, K = topk_weights.shape
    H = expert_out_u16.shape[-1]
    eo = dev_u16_as_bf16(expert_out_u16) if expert_out_u16.size else torch.empty(
        (0, H), dtype=torch.bfloat16, device="cuda")
    y = Guarded((T, H), torch.bfloat16)
    wts = torch.from_numpy(np.ascontiguousarray(topk_weights, np.float32)).cuda()
    ep.ep_combine(eo, lay, wts, y.t, ws)
    torch.cuda.synchronize()
    return bf16_to_u16(y.t), y.canary_ok()


def torch_identity_expert(recv_q: torch.Tensor, recv_s: torch.Tensor) -> torch.Tensor:
    """Stand-in for the expert computation (tests and benchmarks only): dequantise
    E4M3 rows with one fp32 multiply and round to BF16."""
    H = recv_q.shape[-1]
    q = recv_q.view(torch.float8_e4m3fn).to(torch.float32)
    s = recv_s[..., : H // 128].repeat_interleave(128, dim=-1)
    return (q * s).to(torch.bfloat16)
