"""Expert-parallel MoE layer over the ranks of one node (one process per GPU).

Paper review "Breaking the Training Barrier of Billion-Parameter Universal
Machine Learning Interatomic Potentials", section 3.4 (FSEP: experts sharded
over ranks) and section 3.5 (the MoE all-to-all of atom-type-aware FP16
rows).  Rank o holds the weights of experts [o*E/P, (o+1)*E/P) and its own
atoms.  One layer pass:

  forward:  route (local) -> gather counts -> layout -> FP16 pack-and-send to
            the owners -> barrier -> owner: unpack, experts -> return to the
            senders -> barrier -> combine (local)
  VJP:      weighted FP32 send of dY -> barrier -> owner: input VJP of its
            experts -> return -> barrier -> combine (local)

The owner's unpack is fused into the experts' first GEMM: it loads the
received FP16 rows and their scales itself (janus_expert_ffn_fwd_packed).
The return is fused into the experts' last GEMM by default: its epilogue
stores each output row straight into the sender's return buffer through a row
table (janus_ep_return_rows), so the rows cross NVLink as the tiles finish and
no separate copy kernel runs.  fused_return=False keeps the copy kernel
(janus_ep_return) after the GEMM.

Every step is a kernel of libjanus; torch.distributed carries only the
counts, the IPC handles (once) and the phase barriers.  The receive buffers
are allocated once for capacity_factor times a rank's fair share of rows
(N_max*K; the worst case, every rank's rows on one owner, is P times that), so
no step waits for the host to learn a count.  Rows that would land past the
capacity are not sent: the send kernels record a data fault, which `check()`
raises.  With NCCL a barrier
is a one-element all-reduce on the current stream (stream-ordered: every
rank's send kernel has finished before any rank passes it); with gloo it is a
stream synchronize plus a host barrier.
"""
import torch
import torch.distributed as dist

from . import janus as J


class ExpertParallelLayer:
    """Buffers, peer mappings and the ordered calls of one EP layer pass."""

    def __init__(self, n_atoms_max, d, h, n_types, n_experts, top_k, w1_local, w2_local, *,
                 mode=J.JANUS_FFN_3XTF32, group=None, device=None, fused_return=True, capacity_factor=2.0):
        self.group = group
        self.dist = dist.is_available() and dist.is_initialized()
        # without a process group the layer is a single rank owning every expert
        self.world = dist.get_world_size(group) if self.dist else 1
        self.rank = dist.get_rank(group) if self.dist else 0
        if self.world > J.JANUS_EP_MAX_RANKS:
            raise ValueError(f"at most {J.JANUS_EP_MAX_RANKS} ranks (one node)")
        if n_experts % self.world:
            raise ValueError("the number of experts must be a multiple of the number of ranks")
        self.dev = torch.device(device) if device is not None else w1_local.device
        self.d, self.h, self.T, self.E, self.K = d, h, n_types, n_experts, top_k
        self.El = n_experts // self.world
        if w1_local.shape != (self.El, d, h) or w2_local.shape != (self.El, h, d):
            raise ValueError("w1_local / w2_local must hold this rank's E/P experts")
        self.w1, self.w2, self.mode = w1_local, w2_local, mode
        self.fused_return = bool(fused_return)
        # the received FP16 rows go straight into the first GEMM (its
        # tensor-core form needs d % 8 == 0; otherwise they are unpacked first)
        self.fused_unpack = mode == J.JANUS_FFN_FP32_SIMT or d % 8 == 0
        self.nccl = self.dist and dist.get_backend(group) == "nccl"
        # receive capacity: capacity_factor x the fair share (this rank's own
        # routed rows), never more than the worst case (every rank's rows here)
        self.n_atoms_max = int(n_atoms_max)
        rows = max(self.n_atoms_max * top_k, 1)
        if capacity_factor <= 0:
            raise ValueError("capacity_factor must be positive")
        cap = max(1, min(self.world * rows, int(-(-capacity_factor * rows // 1))))
        f32 = dict(dtype=torch.float32, device=self.dev)
        self.cap = cap
        # this library's kernels per forward + VJP: route 4, layout 1, pack 2,
        # expert MLP 2 + 2, FP32 send 1, combine 1 + 1, the unpack 1 (when not
        # fused), and the return table (fused) or the return copy twice; the
        # fused 3xTF32 forward adds W1's split (1) and, from the library's row
        # threshold per local expert (receive capacity) with h % 8 == 0, the
        # FP16 second GEMM's row split (1) and W2's split (1)
        self.launches_per_step = 14 + (0 if self.fused_unpack else 1) + (1 if self.fused_return else 2)
        f16_first = self.fused_unpack and mode == J.JANUS_FFN_3XTF32
        min_rows = J.janus_expert_ffn_f16_min_rows_per_expert()
        self.f16_second = f16_first and h % 8 == 0 and cap >= min_rows * self.El
        self.launches_per_step += (1 if f16_first else 0) + (2 if self.f16_second else 0)
        # the VJP on the FP16 tensor path at the same size: the received
        # gradient rows split into two FP16 terms (row maxima + split), then
        # W2's split, dH, dA's split, W1's split, dA W1^T in place of 2 GEMMs
        self.split_vjp = (mode == J.JANUS_FFN_3XTF32 and d % 8 == 0 and h % 8 == 0
                          and cap >= min_rows * self.El)
        self.launches_per_step += 5 if self.split_vjp else 0
        # both directions on the FP16 path: the forward writes the weights'
        # splits for both (janus_expert_weights_f16, 2 launches in place of
        # the forward's two splits) and the VJP launches none of its own
        self.w16set = None
        if self.f16_second and self.split_vjp:
            self.w16set = torch.empty(J.janus_expert_weights_f16_size(self.El, d, h), dtype=torch.uint8,
                                      device=self.dev)
            self.launches_per_step -= 2
        self.payload = torch.empty((cap, d), dtype=torch.float16, device=self.dev)
        self.row_scale = torch.empty((cap,), **f32)
        self.recv_rows = torch.empty((cap, d), **f32)       # gradients in, outputs out
        self.xd = torch.empty((cap, d), **f32)
        self.act = torch.empty((cap, h), **f32)
        self.yd = torch.empty((cap, d), **f32)
        self.ret = torch.empty((rows, d), **f32)             # this rank's rows coming back
        self.ret_rows = torch.zeros((cap,), dtype=torch.int64, device=self.dev)   # fused-return row table
        if self.split_vjp:
            self.gd16 = torch.empty((2 * cap, d), dtype=torch.float16, device=self.dev)
            self.gd_scale = torch.empty((cap,), **f32)
            self.ident = torch.arange(cap, dtype=torch.int32, device=self.dev)
            self.split_ws = torch.empty(J.janus_dispatch_split_workspace_size(cap), dtype=torch.uint8,
                                        device=self.dev)
            self.vjp_ws = torch.empty(J.janus_expert_ffn_split_workspace_size(cap, self.El, d, h),
                                      dtype=torch.uint8, device=self.dev)
        self.counts_all = torch.empty((self.world, n_experts), dtype=torch.int32, device=self.dev)
        # error word of the sends (both directions): rows past the capacity
        self.send_ws = torch.empty(J.janus_quant_by_type_workspace_size(n_types), dtype=torch.uint8,
                                   device=self.dev)
        self._token = torch.zeros(1, **f32)
        self._opened = []
        self.peer_payload = self._exchange(self.payload)
        self.peer_scale = self._exchange(self.row_scale)
        self.peer_rows = self._exchange(self.recv_rows)
        self.peer_ret = self._exchange(self.ret)

    # -- plumbing ------------------------------------------------------------
    def _exchange(self, t):
        """Device pointers of every rank's copy of buffer t (index = rank)."""
        if self.world == 1:
            return [t.data_ptr()]
        blob = J.janus_ipc_get_handle(t)
        blobs = [None] * self.world
        dist.all_gather_object(blobs, blob, group=self.group)
        ptrs = []
        for r, b in enumerate(blobs):
            if r == self.rank:
                ptrs.append(t.data_ptr())
            else:
                p, off = J.janus_ipc_open_handle(b)
                self._opened.append((p, off))
                ptrs.append(p)
        return ptrs

    def barrier(self):
        """Every rank's work queued so far (its peer stores included) is done
        before any rank's next step runs."""
        if self.world == 1:
            return
        if self.nccl:
            dist.all_reduce(self._token, group=self.group)
        else:
            torch.cuda.current_stream(self.dev).synchronize()
            dist.barrier(group=self.group)

    def _gather_counts(self, counts):
        if self.world == 1:
            self.counts_all[0].copy_(counts)
        elif self.nccl:
            dist.all_gather_into_tensor(self.counts_all, counts, group=self.group)
        else:
            parts = [torch.empty_like(counts.cpu()) for _ in range(self.world)]
            dist.all_gather(parts, counts.cpu(), group=self.group)
            self.counts_all.copy_(torch.stack(parts))

    def check(self):
        """Raise JanusError(JANUS_ERR_DATA) if this rank's sends met a data
        fault since the last forward (bad type ids, non-finite features, or
        rows past an owner's receive capacity).  Synchronises the stream."""
        J.janus_check(self.send_ws)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
        return False

    def close(self):
        torch.cuda.synchronize(self.dev)
        if self.world > 1:
            dist.barrier(group=self.group)      # no rank still writes into a mapping
        for p, off in self._opened:
            J.janus_ipc_close_handle(p, off)
        self._opened = []

    # -- the layer -------------------------------------------------------------
    PHASES_FWD = ("route", "layout", "send", "ffn_fwd", "return", "combine")
    PHASES_VJP = ("send_vjp", "ffn_vjp", "return_vjp", "combine_vjp")

    @staticmethod
    def _mark(events, name, i):
        if events is not None:
            events[name][i].record()

    def forward(self, x, types, gate, events=None):
        """y [N,d] for this rank's atoms (FP16-packed dispatch).  events: an
        optional dict phase -> (start, end) CUDA events to record."""
        if x.shape[0] > self.n_atoms_max:
            raise ValueError("more atoms than the buffers were sized for")
        m = self._mark
        self.x_shape = x.shape
        m(events, "route", 0)
        self.route = J.janus_route(types, gate, self.K)
        m(events, "route", 1)
        m(events, "layout", 0)
        self._gather_counts(self.route["counts"])
        self.layout = J.janus_ep_layout(self.counts_all, self.E, self.cap)
        m(events, "layout", 1)
        m(events, "send", 0)
        J.janus_ep_dispatch_quant(x, types, self.T, self.route, self.layout, self.rank, self.cap,
                                  self.peer_payload, self.peer_scale, workspace=self.send_ws)
        self.barrier()
        m(events, "send", 1)
        recv_off = self.layout[2][self.rank]
        m(events, "ffn_fwd", 0)
        out = dict(out=self.yd)
        if self.fused_return:
            # the table depends only on the layout: the VJP reuses it
            J.janus_ep_return_rows(self.layout, self.rank, self.peer_ret, self.cap, self.d, out=self.ret_rows)
            out = dict(out_rows=self.ret_rows)
        if self.fused_unpack:
            if self.w16set is not None:
                J.janus_expert_weights_f16(self.w1, self.w2, J.JANUS_W16_FWD | J.JANUS_W16_VJP, out=self.w16set)
            J.janus_expert_ffn_fwd_packed(self.payload, self.row_scale, recv_off, self.w1, self.w2, act=self.act,
                                          mode=self.mode, weights16=self.w16set, **out)
        else:
            # the unpacked FP16 rows are exact in TF32: the first GEMM skips their residual
            J.janus_ep_dequant_rows(self.payload, self.row_scale, self.layout, self.rank, out=self.xd)
            J.janus_expert_ffn_fwd_ex(self.xd, recv_off, self.w1, self.w2, act=self.act,
                                      flags=J.JANUS_FFN_X_DEQUANTIZED, mode=self.mode, **out)
        m(events, "ffn_fwd", 1)
        m(events, "return", 0)
        if not self.fused_return:
            J.janus_ep_return(self.yd, self.counts_all, self.layout, self.rank, self.peer_ret)
        self.barrier()
        m(events, "return", 1)
        R = x.shape[0] * self.K
        m(events, "combine", 0)
        y = J.janus_combine(self.ret[:R], self.route["slot_of"], self.K, self.route["topk_weight"])
        m(events, "combine", 1)
        return y

    def vjp(self, g, events=None):
        """dx [N,d] for the upstream gradient g [N,d] of forward's output."""
        m = self._mark
        r = self.route
        m(events, "send_vjp", 0)
        J.janus_ep_dispatch(g, r, self.layout, self.rank, self.cap, self.peer_rows, weighted=True,
                            workspace=self.send_ws)
        self.barrier()
        m(events, "send_vjp", 1)
        recv_off = self.layout[2][self.rank]
        m(events, "ffn_vjp", 0)
        if self.split_vjp:
            # every receive row is split (the ones past this step's rows are
            # never read by the GEMMs); the results go through the return
            # table (fused) or into yd
            J.janus_dispatch_split(self.recv_rows, self.ident, 1, out=self.gd16, row_scale=self.gd_scale,
                                   workspace=self.split_ws)
            out = dict(out_rows=self.ret_rows) if self.fused_return else dict(out=self.yd)
            J.janus_expert_ffn_vjp_split(self.gd16, self.gd_scale, recv_off, self.w1, self.w2, self.act,
                                         weights16=self.w16set, workspace=self.vjp_ws, **out)
        elif self.fused_return:
            J.janus_expert_ffn_vjp_rows(self.xd, self.recv_rows, recv_off, self.w1, self.w2, self.ret_rows,
                                        act=self.act, mode=self.mode)
        else:
            J.janus_expert_ffn_vjp(self.xd, self.recv_rows, recv_off, self.w1, self.w2, act=self.act,
                                   mode=self.mode, out=self.yd)
        m(events, "ffn_vjp", 1)
        m(events, "return_vjp", 0)
        if not self.fused_return:
            J.janus_ep_return(self.yd, self.counts_all, self.layout, self.rank, self.peer_ret)
        self.barrier()
        m(events, "return_vjp", 1)
        R = self.x_shape[0] * self.K
        m(events, "combine_vjp", 0)
        dx = J.janus_combine(self.ret[:R], r["slot_of"], self.K)
        m(events, "combine_vjp", 1)
        return dx
