"""Buffer owner for one single-GPU routing step: torch allocates device memory,
the library's kernels do all the work.

    pipe = RoutingPipeline(N=128, K=2048, E=128, top_k=8, N_out=768, mode="w4a16")
    pipe.quantize_weights(w_f32_expert_slices)      # offline, once
    pipe.x.copy_(...); pipe.routing_map.copy_(...); pipe.router_weights.copy_(...)
    pipe.real_token_count.fill_(real)
    pipe.run()                                      # mask + indices -> GEMV (|| dispatch) -> combine
    pipe.output                                     # bf16 [N, N_out]

Every buffer is allocated once at construction, so ``run`` allocates
nothing and can be captured in a CUDA graph.
"""
from __future__ import annotations

import torch

from . import (MOE_EPI_IDENTITY, MOE_EPI_NONE, MOE_EPI_SCALE, MOE_GEMV_TENSOR_MEMORY,
               MOE_W4A4, MOE_W4A16,
               moe_combine, moe_create_indices, moe_create_indices_workspace_bytes,
               moe_mask_and_create_indices, moe_grouped_gemv_plan,
               moe_grouped_gemv_workspace_bytes,
               moe_dispatch_mxfp4, moe_dispatch_mxfp4_quantize_nvfp4, moe_grouped_gemv_nvfp4,
               moe_mask_padding,
               moe_mxfp4_row_stride, moe_quantize_activations_nvfp4, moe_quantize_weights_nvfp4)

EPILOGUES = {"none": MOE_EPI_NONE, "identity": MOE_EPI_IDENTITY, "scale": MOE_EPI_SCALE}


def _arena_layout(fields, align: int = 256):
    """Byte offsets of the fields (name, shape, dtype), each aligned to
    ``align``; returns (entries, total bytes)."""
    entries, off = [], 0
    for name, shape, dtype in fields:
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        entries.append((name, shape, dtype, off, nbytes))
        off += (nbytes + align - 1) // align * align
    return entries, max(off, align)


def _arena_views(buf: torch.Tensor, entries):
    return {name: buf[off:off + nbytes].view(dtype).view(shape)
            for name, shape, dtype, off, nbytes in entries}


class RoutingPipeline:
    # where run() forks the MXFP4 dispatch onto side_stream in the
    # "routing_first" order: "routing" (after mask + create_indices, beside the
    # GEMV, on SMs its CTAs leave free) or "gemv" (after the GEMV, beside the
    # combine)
    dispatch_fork = "routing"

    def __init__(self, N: int, K: int, E: int, top_k: int, N_out: int, mode: str = "w4a16",
                 epilogue: str = "none", alpha: float = 1.0, tp_rank: int = 0,
                 act_global: float = 1.0, device: str | torch.device = "cuda",
                 recv_capacity: int | None = None, dispatch: bool = True):
        self.N, self.K, self.E, self.top_k, self.N_out = N, K, E, top_k, N_out
        self.mode = mode
        self.gemv_mode = MOE_W4A16 if mode == "w4a16" else MOE_W4A4
        self.epi = EPILOGUES[epilogue]
        self.alpha = float(alpha)
        self.tp_rank = tp_rank
        self.act_global = float(act_global)
        self.dispatch = dispatch
        dev = torch.device(device)
        self.device = dev
        S = N * top_k
        self.S = S
        u8, i32, i64 = torch.uint8, torch.int32, torch.int64
        # inputs: views into one byte arena, so a step's inputs travel from a
        # pinned host mirror (host_inputs()) in a single copy
        # (the routing inputs come first: they can be copied ahead of x)
        self._input_layout = _arena_layout([
            ("routing_map", (N, top_k), i64), ("router_weights", (N, top_k), torch.float32),
            ("real_token_count", (1,), i32), ("x", (N, K), torch.bfloat16)])
        self.routing_bytes = self._input_layout[0][3][3]   # offset of x in the arena
        self.inputs = torch.zeros(self._input_layout[1], dtype=u8, device=dev)
        for name, t in _arena_views(self.inputs, self._input_layout[0]).items():
            setattr(self, name, t)
        # expert library
        self.wq = torch.empty((E, N_out, K // 2), dtype=u8, device=dev)
        self.sfw = torch.empty((E, N_out, K // 16), dtype=u8, device=dev)
        self.w_global = torch.ones(E, dtype=torch.float32, device=dev)
        # step 2
        self.token_expert_order = torch.empty(S, dtype=i32, device=dev)
        self.expert_start_indices = torch.empty(E + 1, dtype=i32, device=dev)
        self.restore_token_order = torch.empty(S, dtype=i32, device=dev)
        self.expert_ids = torch.empty(E, dtype=i32, device=dev)
        self.expert_usage_stats = torch.empty(2, dtype=i32, device=dev)
        self.scales_offset = torch.empty(E + 1, dtype=i32, device=dev)
        self.ws_bytes = moe_create_indices_workspace_bytes(S, E)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=u8, device=dev)
        # step 3
        self.stride = moe_mxfp4_row_stride(K)
        self.recv_capacity = S if recv_capacity is None else recv_capacity
        self.recv_buf = torch.empty((self.recv_capacity, self.stride), dtype=u8, device=dev)
        self.recv_counts = torch.empty(E, dtype=i32, device=dev)
        # step 4
        if self.gemv_mode == MOE_W4A4:
            self.xq = torch.empty((N, K // 2), dtype=u8, device=dev)
            self.sfa = torch.empty((N, K // 16), dtype=u8, device=dev)
        else:
            self.xq = self.sfa = None
        self.expert_out = torch.zeros((N, top_k, N_out), dtype=torch.bfloat16, device=dev)
        # the GEMV's workspace: its grouping (when handed the map alone) and, for W4A16
        # in the tensor-memory variant, the activations converted once
        self.gemv_ws_bytes = moe_grouped_gemv_workspace_bytes(N, top_k, E, K)
        self.gemv_ws = torch.empty(max(self.gemv_ws_bytes, 256), dtype=u8, device=dev)
        # Step order of run():
        #   "gemv_groups"   mask -> GEMV on the routing map (the GEMV groups the
        #                   pairs in-kernel) -> combine; create_indices and the
        #                   dispatch on the side stream
        #   "routing_first" mask + create_indices -> GEMV on the grouping ->
        #                   combine; the dispatch on the side stream
        # The first is taken when the GEMV variant for these shapes groups the
        # map itself (decode-sized W4A16), so grouping is off its critical path.
        _, in_kernel = moe_grouped_gemv_plan(self.gemv_mode, N, top_k, E, N_out, K)
        self.order = "gemv_groups" if in_kernel else "routing_first"
        # the variant the routing_first order's GEMV (grouping given) runs
        self.gemv_variant, _ = moe_grouped_gemv_plan(self.gemv_mode, N, top_k, E, N_out, K,
                                                     grouping_given=True)
        # W4A4 in the "routing_first" order: the MXFP4 dispatch and the NVFP4
        # activation quantisation as one kernel (one read of x) before the GEMV
        self.fuse_dispatch_quant = self.gemv_mode == MOE_W4A4 and dispatch
        # step 5
        self.output = torch.empty((N, N_out), dtype=torch.bfloat16, device=dev)
        # timing events go on a side stream, so no event sits between two kernels
        # of the main stream (which would cut their programmatic dependency)
        self._timer = torch.cuda.Stream(device=dev)
        # recorded on the side stream before a dispatch forked after the routing
        # kernel: a graph's event-record node there turns the dispatch's
        # programmatic dependency into a plain one, so its CTAs do not take SMs
        # before the GEMV's.  Kept alive with the pipeline (captured graphs use it).
        self._dispatch_marker = torch.cuda.Event(external=True)

    def host_inputs(self):
        """A pinned host byte buffer laid out like ``inputs`` and its typed
        views (x, routing_map, router_weights, real_token_count):
        ``pipe.inputs.copy_(buf, non_blocking=True)`` moves a whole step's
        inputs in one transfer."""
        buf = torch.zeros(self._input_layout[1], dtype=torch.uint8, pin_memory=True)
        return buf, _arena_views(buf, self._input_layout[0])

    # ------------------------------------------------------------ weights
    def quantize_weights(self, w_f32: torch.Tensor, expert_base: int = 0, stream=None):
        """Quantise fp32 weights [e, N_out, K] (device) into experts [base, base + e)."""
        e = w_f32.shape[0]
        assert w_f32.shape[1:] == (self.N_out, self.K) and w_f32.is_cuda
        w = w_f32.contiguous()
        moe_quantize_weights_nvfp4(w, e, self.N_out, self.K, self.wq[expert_base:expert_base + e],
                                   self.sfw[expert_base:expert_base + e],
                                   self.w_global[expert_base:expert_base + e], stream)

    # ------------------------------------------------------------ steps
    def mask(self, stream=None):
        moe_mask_padding(self.routing_map, self.N, self.top_k, self.real_token_count,
                         self.tp_rank, stream)

    def create_indices(self, stream=None):
        moe_create_indices(self.routing_map, self.S, self.E, self.token_expert_order,
                           self.expert_start_indices, self.restore_token_order, self.expert_ids,
                           self.expert_usage_stats, self.scales_offset, self.workspace,
                           self.ws_bytes, stream)

    def mask_and_create_indices(self, stream=None):
        moe_mask_and_create_indices(self.routing_map, self.N, self.top_k, self.real_token_count,
                                    self.tp_rank, self.E, self.token_expert_order,
                                    self.expert_start_indices, self.restore_token_order,
                                    self.expert_ids, self.expert_usage_stats, self.scales_offset,
                                    self.workspace, self.ws_bytes, stream)

    def dispatch_mxfp4(self, stream=None):
        moe_dispatch_mxfp4(self.x, self.N, self.K, self.top_k, self.E, self.restore_token_order,
                           self.expert_start_indices, self.expert_ids, self.expert_usage_stats,
                           self.recv_buf, self.recv_capacity, self.recv_counts, stream)

    def dispatch_quantize(self, stream=None):
        """The MXFP4 dispatch and the NVFP4 activation quantisation from one
        read of x (W4A4)."""
        moe_dispatch_mxfp4_quantize_nvfp4(
            self.x, self.N, self.K, self.top_k, self.E, self.restore_token_order,
            self.expert_start_indices, self.expert_ids, self.expert_usage_stats, self.recv_buf,
            self.recv_capacity, self.recv_counts, self.act_global, self.xq, self.sfa, stream)

    def quantize_activations(self, stream=None):
        moe_quantize_activations_nvfp4(self.x, self.N, self.K, self.act_global, self.xq,
                                       self.sfa, stream)

    def gemv(self, stream=None):
        """The GEMV on the step-2 grouping."""
        act = self.x if self.gemv_mode == MOE_W4A16 else self.xq
        moe_grouped_gemv_nvfp4(self.gemv_mode, act, self.sfa, self.act_global, self.routing_map,
                               self.N, self.top_k, self.wq, self.sfw, self.w_global, self.E,
                               self.N_out, self.K, self.token_expert_order,
                               self.expert_start_indices, self.expert_ids,
                               self.expert_usage_stats, self.expert_out, workspace=self.gemv_ws,
                               ws_bytes=self.gemv_ws_bytes, stream=stream)

    def gemv_on_map(self, stream=None):
        """The GEMV on the routing map alone (it groups the pairs itself)."""
        act = self.x if self.gemv_mode == MOE_W4A16 else self.xq
        moe_grouped_gemv_nvfp4(self.gemv_mode, act, self.sfa, self.act_global, self.routing_map,
                               self.N, self.top_k, self.wq, self.sfw, self.w_global, self.E,
                               self.N_out, self.K, out=self.expert_out, workspace=self.gemv_ws,
                               ws_bytes=self.gemv_ws_bytes, stream=stream)

    def combine(self, stream=None):
        moe_combine(self.expert_out, self.router_weights, self.routing_map, self.N, self.top_k,
                    self.N_out, self.E, self.epi, self.alpha, self.output, stream)

    def run(self, stream=None, gemv_events=None, side_stream=None, x_ready=None):
        """All steps in order (see ``order``).  ``gemv_events`` = (start, end)
        CUDA events recorded around the GEMV launch (from a side stream), for
        per-kernel timing.  With ``side_stream``, the work whose outputs neither
        the GEMV nor the combine reads -- the MXFP4 dispatch, and in the
        "gemv_groups" order create_indices too -- runs there and joins at the
        end.  ``x_ready`` (a CUDA event) holds back the steps that read the
        activations -- dispatch, activation quantisation, GEMV -- until x has
        arrived; mask and create_indices run before it."""
        main = stream if stream is not None else torch.cuda.current_stream()
        if self.order == "gemv_groups":
            self._run_gemv_groups(main, gemv_events, side_stream, x_ready)
        else:
            self._run_routing_first(main, gemv_events, side_stream, x_ready)
        if gemv_events is not None:
            timer_done = torch.cuda.Event()
            timer_done.record(self._timer)
            main.wait_event(timer_done)

    def _run_gemv_groups(self, main, gemv_events, side_stream, x_ready):
        self.mask(main)
        join = None
        if side_stream is not None:
            fork = torch.cuda.Event()
            fork.record(main)
            side_stream.wait_event(fork)
            self.create_indices(side_stream)
            if self.dispatch:
                if x_ready is not None:
                    side_stream.wait_event(x_ready)
                self.dispatch_mxfp4(side_stream)
            join = torch.cuda.Event()
            join.record(side_stream)
        else:
            self.create_indices(main)
        if x_ready is not None:
            main.wait_event(x_ready)
        if side_stream is None and self.dispatch:
            self.dispatch_mxfp4(main)
        if self.gemv_mode == MOE_W4A4:
            self.quantize_activations(main)
        if gemv_events is not None:
            self._mark(main, gemv_events[0])
        self.gemv_on_map(main)
        if gemv_events is not None:
            self._mark(main, gemv_events[1])
        self.combine(main)
        if join is not None:
            main.wait_event(join)

    def _run_routing_first(self, main, gemv_events, side_stream, x_ready):
        self.mask_and_create_indices(main)
        if self.fuse_dispatch_quant:
            if x_ready is not None:
                main.wait_event(x_ready)
            self.dispatch_quantize(main)
            if gemv_events is not None:
                self._mark(main, gemv_events[0])
            self.gemv(main)
            if gemv_events is not None:
                self._mark(main, gemv_events[1])
            self.combine(main)
            return
        forked = self.dispatch and side_stream is not None
        early = forked and self.dispatch_fork == "routing"
        if early:
            fork = torch.cuda.Event()
            fork.record(main)
            side_stream.wait_event(fork)
            if x_ready is not None:
                side_stream.wait_event(x_ready)
            self._dispatch_marker.record(side_stream)
            self.dispatch_mxfp4(side_stream)
            join = torch.cuda.Event()
            join.record(side_stream)
        if x_ready is not None:
            main.wait_event(x_ready)
        if self.dispatch and not forked:
            self.dispatch_mxfp4(main)
        if self.gemv_mode == MOE_W4A4:
            self.quantize_activations(main)
        if gemv_events is not None:
            self._mark(main, gemv_events[0])
        self.gemv(main)
        if gemv_events is not None:
            self._mark(main, gemv_events[1])
        if forked and not early:
            fork = torch.cuda.Event()
            fork.record(main)
            side_stream.wait_event(fork)
            self.dispatch_mxfp4(side_stream)
            join = torch.cuda.Event()
            join.record(side_stream)
        self.combine(main)
        if forked:
            main.wait_event(join)

    def _mark(self, main, event):
        """Record ``event`` once everything enqueued on ``main`` so far has run,
        from the side timer stream."""
        here = torch.cuda.Event()
        here.record(main)
        self._timer.wait_event(here)
        event.record(self._timer)

    def kernel_steps(self):
        """(name, step) for every step of run(), in order, serialised on one
        stream; each step takes the stream to enqueue on.  For per-kernel
        timing."""
        if self.order == "gemv_groups":
            steps = [("mask", self.mask), ("create_indices", self.create_indices)]
        else:
            steps = [("mask+create_indices", self.mask_and_create_indices)]
        if self.order == "routing_first" and self.fuse_dispatch_quant:
            steps.append(("dispatch+quant_act", self.dispatch_quantize))
        else:
            if self.dispatch:
                steps.append(("dispatch_mxfp4", self.dispatch_mxfp4))
            if self.gemv_mode == MOE_W4A4:
                steps.append(("quant_act_nvfp4", self.quantize_activations))
        gemv = self.gemv_on_map if self.order == "gemv_groups" else self.gemv
        steps.append(("grouped_gemv", gemv))
        steps.append(("combine", self.combine))
        return steps

    def launches_per_run(self) -> int:
        """Kernel launches of one run() (an estimate; bench.py counts the
        kernel nodes of the captured graph)."""
        ci = 1 if self.S <= 16384 else 2
        if self.order == "gemv_groups":
            n = 1 + ci + 1                       # mask, create_indices, GEMV (groups in-kernel)
        else:
            n = (1 if self.S <= 1024 else 1 + ci) + 1
            if self.gemv_mode == MOE_W4A16 and self.gemv_variant == MOE_GEMV_TENSOR_MEMORY:
                n += 1                           # the activations' fp16 conversion
        if self.order == "routing_first" and self.fuse_dispatch_quant:
            n += 1
        else:
            n += 1 if self.dispatch else 0
            n += 1 if self.gemv_mode == MOE_W4A4 else 0
        return n + 1                             # combine
