"""Expert parallelism for the MoE layer forward pass.

"Kimi K3: Open Frontier Intelligence", section "Systems Optimization, Load
Balancing, and Post-Training Alignment", splits the routed experts over ranks:
rank g of a group of G owns experts [g E/G, (g+1) E/G), every rank routes its
own tokens, and each dispatched (token, expert) row travels to the rank that
owns its expert, through that expert's feed-forward block, and back, where the
token's k rows are combined. The page sizes each rank's traffic as a fixed
S x K rows so that the exchange needs no host synchronisation; that is the
"capacity" mode here.

One forward pass on each rank, in order (every rank takes the same collective
steps in the same order):
  1. route and build the dispatch tables (this library's kernels);
  2. exchange the per-expert row counts: one all-to-all of G x E/G int32;
  3. exchange the rows: one all-to-all (exact mode: of exactly the rows each
     pair has, whose sizes the host reads once; capacity mode: C rows per pair,
     no host read, padding rows zero);
  4. on the owner: gather the received rows into one expert-major block,
     run the grouped SwiGLU feed-forward of the local experts, gather the
     results back into arrival order;
  5. send the results back: one all-to-all of the same shape as step 3;
  6. combine each token's k rows in slot order (this library's kernel).

The index bookkeeping between the steps (where each row goes) is integer
arithmetic on O(T k) int32 values on the device (torch tensor ops, no host
read except exact mode's split sizes); every row copy, the router, the GEMMs
and the combine run in this library's kernels, through `CudaOps`. Transport is
torch.distributed (NCCL on GPUs). No TMA load in this path reads another GPU's
memory: rows arrive in this GPU's own buffers through the collective.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist


class CudaOps:
    """The local steps, on this library's CUDA kernels (the product path)."""

    ffn_dtype = torch.bfloat16  # dtype of the expert feed-forward's output rows

    def __init__(self):
        from . import _lib
        self._lib = _lib

    def route(self, x, W_router, bias, k):
        return self._lib.moe_route(x, W_router, bias, k)

    def dispatch(self, x, idx, E):
        """(offsets [E+1], perm_token [T k], inv_perm [T, k]) int32, no row copy."""
        offsets, perm, inv, _ = self._lib.moe_permute(x, idx, E, with_rows=False)
        return offsets, perm, inv

    def gather(self, src, rows):
        return self._lib.moe_gather_rows(src, rows)

    def expert_ffn(self, x_rows, offsets, W_gate_up, W_down):
        _, y = self._lib.moe_expert_ffn(x_rows, offsets, W_gate_up, W_down)
        return y

    def combine(self, y_rows, inv, w):
        return self._lib.moe_unpermute(y_rows, inv, w)


@dataclass
class EPStats:
    """Device tensors describing one pass (read them only when needed: reading
    synchronises). send_rows / recv_rows [G]: rows this rank sent to / received
    from each rank; overflow: 1 if capacity mode dropped a row (its
    contribution is then missing from `out`), else 0."""
    send_rows: torch.Tensor
    recv_rows: torch.Tensor
    overflow: torch.Tensor


def _exclusive_cumsum(v: torch.Tensor) -> torch.Tensor:
    c = torch.cumsum(v, 0)
    return c - v


def _a2a(out: torch.Tensor, inp: torch.Tensor, group, out_splits=None, in_splits=None):
    """all_to_all_single moving raw rows: bf16 rows travel as float16 bit
    patterns (no arithmetic is applied to them), which every backend carries."""
    if inp.dtype == torch.bfloat16:
        out_v, in_v = out.view(torch.float16), inp.view(torch.float16)
    else:
        out_v, in_v = out, inp
    dist.all_to_all_single(out_v, in_v, output_split_sizes=out_splits, input_split_sizes=in_splits, group=group)
    return out


def block_maps(cnt: torch.Tensor, C: Optional[int]):
    """Index maps between the arrival order and the expert-major order of the
    rows an owner receives.

    cnt [G, E_loc]: rows source s sent for local expert e (int64). Arrival
    order: source-major blocks (source s at s * C with capacity C, else packed
    back to back), each block ordered by local expert. Expert-major order:
    expert e's rows from source 0, then source 1, ...
    Returns (local_offsets [E_loc + 1] int32, src_of_dst [n_dst] int32 (the
    arrival row of each expert-major row, -1 past the last real row),
    dst_of_src [n_src] int32 (the expert-major row of each arrival row, -1 for
    padding)), with n_dst = n_src = G * C in capacity mode, sum(cnt) otherwise."""
    G, E_loc = cnt.shape
    dev = cnt.device
    per_src = cnt.sum(1)
    if C is None:
        src_base = _exclusive_cumsum(per_src)
        n = int(per_src.sum().item()) if cnt.numel() else 0
        n_src = n_dst = n
    else:
        src_base = torch.arange(G, device=dev, dtype=torch.int64) * C
        n_src = n_dst = G * C
    src_start = src_base[:, None] + (torch.cumsum(cnt, 1) - cnt)   # [G, E_loc] arrival row of block (s, e)
    cnt_em = cnt.t().contiguous()                                  # [E_loc, G], expert-major blocks
    dst_start_em = _exclusive_cumsum(cnt_em.flatten()).view(E_loc, G)
    per_exp = cnt.sum(0)
    local_offsets = torch.zeros(E_loc + 1, dtype=torch.int64, device=dev)
    local_offsets[1:] = torch.cumsum(per_exp, 0)
    total = local_offsets[-1]

    # expert-major row i -> block (e, s) -> arrival row
    i = torch.arange(n_dst, dtype=torch.int64, device=dev)
    starts_em = dst_start_em.flatten()
    b = torch.searchsorted(starts_em, i, right=True) - 1
    b = b.clamp(min=0)
    e_i, s_i = b // G, b % G
    src_of_dst = src_start[s_i, e_i] + (i - starts_em[b])
    src_of_dst = torch.where(i < total, src_of_dst, torch.full_like(src_of_dst, -1))

    # arrival row r -> block (s, e) -> expert-major row
    r = torch.arange(n_src, dtype=torch.int64, device=dev)
    if C is None:
        starts_sm = src_start.flatten()
        b2 = (torch.searchsorted(starts_sm, r, right=True) - 1).clamp(min=0)
        s_r, e_r = b2 // E_loc, b2 % E_loc
        valid = r < total
    else:
        s_r = r // C
        within = r - s_r * C
        ends = torch.cumsum(cnt, 1)                                # [G, E_loc] inclusive ends within each source
        e_r = torch.searchsorted(ends, within.view(G, C), right=True).view(-1).clamp(max=E_loc - 1)
        valid = within < per_src[s_r]
    dst_of_src = dst_start_em[e_r, s_r] + (r - src_start[s_r, e_r])
    dst_of_src = torch.where(valid, dst_of_src, torch.full_like(dst_of_src, -1))
    return local_offsets.to(torch.int32), src_of_dst.to(torch.int32), dst_of_src.to(torch.int32)


def ep_forward(x: torch.Tensor, W_router: torch.Tensor, router_bias: Optional[torch.Tensor],
               W_gate_up_local: torch.Tensor, W_down_local: torch.Tensor, k: int, group=None,
               capacity: Optional[int] = None, mode: str = "exact", ops=None):
    """The MoE layer forward pass with the experts split over the ranks of
    `group`: this rank holds experts [g E_loc, (g + 1) E_loc) as
    W_gate_up_local [E_loc, d, 2f] and W_down_local [E_loc, f, d], and the
    full router W_router [d, E]; x [T, d] are this rank's tokens (every rank
    the same T in capacity mode). Returns (out [T, d], EPStats).

    mode "exact": rows exchanged exactly (one host read of the split sizes).
    mode "capacity": C = `capacity` rows per (source, owner) pair (default
    T * min(k, E_loc), which no routing can exceed); no host read, so the pass
    can be captured in a CUDA graph; rows beyond C are dropped and flagged."""
    ops = ops or CudaOps()
    G = dist.get_world_size(group)
    g = dist.get_rank(group)
    E = W_router.shape[1]
    if E % G:
        raise ValueError(f"E = {E} experts do not split evenly over {G} ranks")
    E_loc = E // G
    if W_gate_up_local.shape[0] != E_loc or W_down_local.shape[0] != E_loc:
        raise ValueError(f"rank {g} must hold {E_loc} experts")
    T, d = x.shape
    dev = x.device

    # 1. route and dispatch tables
    idx, w = ops.route(x, W_router, router_bias, k)
    offsets, perm_token, inv_perm = ops.dispatch(x, idx, E)
    off64 = offsets.to(torch.int64)
    bounds = off64[::E_loc]                                        # [G + 1]
    send_rows = bounds[1:] - bounds[:-1]
    cnt_send = (off64[1:] - off64[:-1]).view(G, E_loc)

    if mode == "capacity":
        C = int(capacity) if capacity is not None else T * min(k, E_loc)
        if C < 1:
            raise ValueError("capacity must be at least 1")
        # clamp each destination's rows to C (dropped rows are flagged)
        ends = torch.cumsum(cnt_send, 1)
        cnt_send = (ends.clamp(max=C) - (ends - cnt_send).clamp(max=C)).clamp(min=0)
        overflow = (send_rows > C).any().to(torch.int32)
    elif mode == "exact":
        C = None
        overflow = torch.zeros((), dtype=torch.int32, device=dev)
    else:
        raise ValueError(f"unknown mode {mode!r}")

    # 2. per-expert counts
    cnt_recv = torch.empty_like(cnt_send)
    _a2a(cnt_recv, cnt_send.contiguous(), group)
    recv_rows = cnt_recv.sum(1)

    # 3. rows out: slot (destination g', i) holds x_perm row bounds[g'] + i,
    #    read straight from x through perm_token (no x_perm copy)
    if C is None:
        splits = torch.stack([send_rows, recv_rows]).cpu()
        s_split, r_split = splits[0].tolist(), splits[1].tolist()
        send_buf = ops.gather(x, perm_token)                      # = x_perm, destination-major already
        recv_buf = torch.empty(sum(r_split), d, dtype=x.dtype, device=dev)
        _a2a(recv_buf, send_buf, group, r_split, s_split)
    else:
        slot = torch.arange(G * C, dtype=torch.int64, device=dev)
        dst_g, i = slot // C, slot % C
        row = bounds[dst_g] + i
        live = i < send_rows[dst_g].clamp(max=C)
        src_tok = torch.where(live, perm_token.to(torch.int64)[row.clamp(max=max(T * k - 1, 0))],
                              torch.full_like(row, -1))
        send_buf = ops.gather(x, src_tok.to(torch.int32))
        recv_buf = torch.empty(G * C, d, dtype=x.dtype, device=dev)
        _a2a(recv_buf, send_buf, group)

    # 4. owner: expert-major block, grouped feed-forward, back to arrival order
    local_offsets, src_of_dst, dst_of_src = block_maps(cnt_recv, C)
    if src_of_dst.numel():
        x_loc = ops.gather(recv_buf, src_of_dst)
        y_loc = ops.expert_ffn(x_loc, local_offsets, W_gate_up_local, W_down_local)
        y_recv = ops.gather(y_loc, dst_of_src)
    else:
        y_recv = torch.empty(0, d, dtype=ops.ffn_dtype, device=dev)   # this rank owns no received row

    # 5. results back, into the sender's slots
    if C is None:
        y_back = torch.empty(T * k, d, dtype=y_recv.dtype, device=dev)
        _a2a(y_back, y_recv, group, s_split, r_split)
        inv_ep, w_eff = inv_perm, w
    else:
        y_back = torch.empty(G * C, d, dtype=y_recv.dtype, device=dev)
        _a2a(y_back, y_recv, group)
        # pair (t, j) sits in slot g' C + (inv_perm - bounds[g']); a dropped
        # pair (local index >= C) keeps weight 0 on slot g' C
        inv64 = inv_perm.to(torch.int64)
        g_pair = idx.to(torch.int64) // E_loc
        local = inv64 - bounds[g_pair]
        kept = local < C
        inv_ep = (g_pair * C + torch.where(kept, local, torch.zeros_like(local))).to(torch.int32)
        w_eff = torch.where(kept, w, torch.zeros_like(w))

    # 6. combine
    out = ops.combine(y_back, inv_ep.contiguous(), w_eff.contiguous())
    return out, EPStats(send_rows=send_rows, recv_rows=recv_rows, overflow=overflow)
