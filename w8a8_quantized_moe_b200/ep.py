"""Expert-parallel W8A8 MoE layer: one rank per GPU over ``torch.distributed``.

"Day0 adaptation of ultra-large model inference" (ruibaoantu.com), section 3:
the experts are spread over the GPUs and each layer moves its tokens with one
All-to-All each way; section 4: gate -> sort -> All-to-All -> grouped GEMM ->
reverse All-to-All -> un-sort -> weighted sum.

Rank g holds a contiguous range of the E experts.  Each rank routes and
quantises its own tokens (``moe_w8a8_ep_dispatch``), sends every kept
(token, slot) row to the rank that holds its expert, runs its experts on the
rows it receives (``moe_w8a8_ep_experts``), returns each output row to its
sender, and sums its tokens' slots in slot order (``moe_w8a8_ep_combine``).
Every rank's output equals the single-GPU layer on that rank's tokens.

The exchange is ``all_to_all_single`` of the process group (NCCL over
NVLink/NVSwitch on GPUs, gloo on CPU for the tests), in one of two forms:

- counted (default): split sizes follow the routing; the per-peer row counts
  are formed on the device from the row offsets, exchanged, and read by the
  host together, once per layer;
- fixed blocks (``block_tokens=B``, every rank's T <= B): each rank sends
  every peer one block of B k + 1 rows, a header row holding the count and
  then the rows (``moe_w8a8_ep_pack``), and gets one output block back, so
  both All-to-Alls have sizes known in advance and no count reaches the host;
  the experts read the counts on the device.  Worst-case bytes on the links
  for no host round trip: the form for decode-sized batches.

All arithmetic of the layer runs in the library's kernels; this module moves
buffers and picks split sizes.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

import w8a8_quantized_moe_b200 as M


def equal_expert_ranges(n_experts: int, world: int) -> list[tuple[int, int]]:
    """(first expert, count) per rank: world equal contiguous ranges."""
    if world <= 0 or n_experts % world:
        raise ValueError(f"{n_experts} experts do not split evenly over {world} ranks")
    n = n_experts // world
    return [(g * n, n) for g in range(world)]


def prepare_expert_shard(cfg: M.moe_w8a8_config, expert_first: int, w_gate, w_up, w_down, w_router,
                         act_absmax, group=None) -> M.Weights:
    """Prepare this rank's experts.  The smoothing statistic aw is the maximum
    over ALL experts of the layer, so the per-rank maxima are all-reduced
    before the scales are formed; every rank then holds the same s.  Runs on
    torch's current stream, the stream the all-reduce is ordered with."""
    aw = torch.empty(cfg.d, dtype=torch.float32, device=w_gate.device)
    M.moe_w8a8_gateup_absmax(cfg, w_gate, w_up, aw)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(aw, op=dist.ReduceOp.MAX, group=group)
    return M.moe_w8a8_prepare_shard(cfg, expert_first, w_gate, w_up, w_down, w_router, act_absmax, aw)


class LibraryStages:
    """The three compute steps of one rank, on the library's kernels.  They run
    on torch's current stream, the stream the collectives are ordered with."""

    def __init__(self, w: M.Weights):
        c = w.cfg
        self.w = w
        self.d, self.k, self.E = c.d, c.top_k, c.n_experts
        self.row_bytes = M.moe_w8a8_ep_row_bytes(w)
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.out_dtype = torch.bfloat16 if c.out_dtype == M.MOE_BF16 else torch.float32

    def dispatch_workspace(self, T: int) -> int:
        return M.moe_w8a8_ep_dispatch_workspace_size(self.w, T)

    def experts_workspace(self, R: int) -> int:
        return M.moe_w8a8_ep_experts_workspace_size(self.w, R)

    def dispatch(self, x, T, router_bias, router_logits, send, offsets, ws):
        M.moe_w8a8_ep_dispatch(self.w, x, T, router_bias, router_logits, send, offsets, ws)

    def experts(self, recv, R, o_rows, ws):
        M.moe_w8a8_ep_experts(self.w, recv, R, o_rows, ws)

    def combine(self, o_rows, T, y, ws):
        M.moe_w8a8_ep_combine(self.w, o_rows, T, y, ws)

    # fixed-block exchange
    def block_rows(self, B):
        return M.moe_w8a8_ep_block_rows(self.w, B)

    def pack(self, send, offsets, rank_first, B, blocks):
        M.moe_w8a8_ep_pack(self.w, send, offsets, rank_first, B, blocks)

    def experts_blocked_workspace(self, world, B):
        return M.moe_w8a8_ep_experts_blocked_workspace_size(self.w, world, B)

    def experts_blocked(self, blocks, world, B, o_blocks, ws):
        M.moe_w8a8_ep_experts_blocked(self.w, blocks, world, B, o_blocks, ws)

    def combine_blocked(self, o_blocks, T, rank_first, B, y, ws):
        M.moe_w8a8_ep_combine_blocked(self.w, o_blocks, T, rank_first, B, y, ws)


class ExpertParallelMoE:
    """One rank of the expert-parallel layer.

    stages        the compute steps (``LibraryStages`` on a GPU)
    ranges        (first expert, count) of every rank, contiguous and
                  ascending; equal ranges by default
    block_tokens  None: the counted exchange; B: the fixed-block exchange,
                  every rank's T <= B (all ranks must pass the same B)
    """

    def __init__(self, stages, group=None, ranges=None, block_tokens=None):
        self.stages = stages
        if block_tokens is not None and block_tokens < 1:
            raise ValueError("block_tokens must be at least 1")
        self.block_tokens = block_tokens
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.ranges = equal_expert_ranges(stages.E, self.world) if ranges is None else list(ranges)
        if len(self.ranges) != self.world:
            raise ValueError("one expert range per rank")
        nxt = 0
        for first, n in self.ranges:
            if first != nxt or n <= 0:
                raise ValueError("expert ranges must be contiguous, ascending and cover every expert")
            nxt = first + n
        if nxt != stages.E:
            raise ValueError("expert ranges must cover every expert")
        self._bufs: dict[str, torch.Tensor] = {}
        self.last_rows = (0, 0)   # rows sent, rows received by the last counted forward
        self._rank_first = [first for first, _ in self.ranges] + [stages.E]
        # row-offset indices of each destination's first expert and one past its last
        self._lo = torch.tensor([first for first, _ in self.ranges], dtype=torch.long, device=stages.device)
        self._hi = torch.tensor([first + n for first, n in self.ranges], dtype=torch.long, device=stages.device)

    def _buf(self, name: str, n: int, dtype) -> torch.Tensor:
        """A cached flat buffer of at least n elements (grown on demand)."""
        b = self._bufs.get(name)
        if b is None or b.numel() < n or b.dtype != dtype:
            b = torch.empty(max(n, 1), dtype=dtype, device=self.stages.device)
            self._bufs[name] = b
        return b[:n]

    def forward(self, x, T: int, router_bias=None, router_logits=None, y=None):
        if self.block_tokens is not None:
            return self._forward_blocked(x, T, router_bias, router_logits, y)
        st = self.stages
        k, E, d, rb = st.k, st.E, st.d, st.row_bytes
        send = self._buf("send", T * k * rb, torch.uint8)
        offsets = self._buf("offsets", E + 1, torch.int32)
        ws_route = self._buf("ws_route", st.dispatch_workspace(T), torch.uint8)
        st.dispatch(x, T, router_bias, router_logits, send, offsets, ws_route)

        # rows per destination (the rows of its experts, contiguous in `send`),
        # exchanged on the device; the host reads sent and received counts at once
        cnt_send = (offsets[self._hi] - offsets[self._lo]).to(torch.int64)
        cnt_recv = torch.empty_like(cnt_send)
        dist.all_to_all_single(cnt_recv, cnt_send, group=self.group)
        counts = torch.cat([cnt_send, cnt_recv]).cpu().tolist()
        send_rows, recv_rows = counts[:self.world], counts[self.world:]
        R_send, R_recv = sum(send_rows), sum(recv_rows)

        recv = self._buf("recv", R_recv * rb, torch.uint8)
        dist.all_to_all_single(recv, send[:R_send * rb], [r * rb for r in recv_rows],
                               [s * rb for s in send_rows], group=self.group)
        o_recv = self._buf("o_recv", R_recv * d, torch.float32)
        ws_exp = self._buf("ws_experts", st.experts_workspace(R_recv), torch.uint8)
        st.experts(recv, R_recv, o_recv.view(R_recv, d), ws_exp)

        # every output row back to the rank and position it came from
        o_back = self._buf("o_back", R_send * d, torch.float32)
        dist.all_to_all_single(o_back, o_recv, [s * d for s in send_rows], [r * d for r in recv_rows],
                               group=self.group)
        if y is None:
            y = torch.empty((T, d), dtype=st.out_dtype, device=st.device)
        st.combine(o_back.view(R_send, d), T, y, ws_route)
        self.last_rows = (R_send, R_recv)
        return y

    def _forward_blocked(self, x, T: int, router_bias, router_logits, y):
        """The fixed-block exchange: nothing of this forward is read by the host."""
        st = self.stages
        B = self.block_tokens
        if T > B:
            raise ValueError(f"T={T} exceeds the exchange's block of {B} tokens")
        k, E, d, rb, G = st.k, st.E, st.d, st.row_bytes, self.world
        rows = st.block_rows(B)
        send = self._buf("send", B * k * rb, torch.uint8)
        offsets = self._buf("offsets", E + 1, torch.int32)
        ws_route = self._buf("ws_route", st.dispatch_workspace(B), torch.uint8)
        st.dispatch(x, T, router_bias, router_logits, send, offsets, ws_route)
        blocks = self._buf("blocks", G * rows * rb, torch.uint8)
        st.pack(send, offsets, self._rank_first, B, blocks)
        recv = self._buf("recv_blocks", G * rows * rb, torch.uint8)
        dist.all_to_all_single(recv, blocks, group=self.group)            # one block per peer each way
        o_blocks = self._buf("o_blocks", G * rows * d, torch.float32)
        ws_exp = self._buf("ws_experts_blocked", st.experts_blocked_workspace(G, B), torch.uint8)
        st.experts_blocked(recv, G, B, o_blocks, ws_exp)
        o_back = self._buf("o_back_blocks", G * rows * d, torch.float32)
        dist.all_to_all_single(o_back, o_blocks, group=self.group)
        if y is None:
            y = torch.empty((T, d), dtype=st.out_dtype, device=st.device)
        st.combine_blocked(o_back, T, self._rank_first, B, y, ws_route)
        self.last_rows = (None, None)
        return y
