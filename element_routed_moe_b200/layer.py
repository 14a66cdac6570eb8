"""One element-routed MoE layer on one GPU: forward and input VJP through the
C ABI, with preallocated buffers.

Sources: paper review "Breaking the Training Barrier of Billion-Parameter
Universal Machine Learning Interatomic Potentials" sections 3.1-3.5 (static
per-element routing, Linear-SiLU-Linear experts, forces by autodiff, FP16
packing of the dispatch, edge aggregation in front of the MoE block) and
"MatRIS-MoE与Janus框架" section 3.2 (gate-weighted sum of the experts).

One pass, all on the current stream:
    [edge_aggregate]  X = segment sums of the edge messages (row_ptr given)
    route             per-type top-K, counts, offsets, permutation
    dispatch          Xd = X rows in expert order   (or FP16 pack, fed to the GEMM as it is)
    ffn_fwd           Yd = silu(Xd W1[e]) W2[e]      (a saved)
    combine           Y  = sum_k w * Yd
    dispatch_w        Gd = w * G rows in expert order
    ffn_vjp           dXd = ((Gd W2^T) * silu'(a)) W1^T
    combine_vjp       dX = sum_k dXd

In 3xTF32 mode the expert MLP runs on the FP16 tensor path where it pays:
FP16-packed rows always go to janus_expert_ffn_fwd_packed as they are (its
first GEMM on kind::f16); with at least SPLIT_MIN_ROWS_PER_EXPERT routed rows
per expert (and d, h multiples of 8) unpacked rows are dispatched as two FP16
terms with a per-row scale (janus_dispatch_split) for
janus_expert_ffn_fwd_split, the gradient's weighted dispatch is split the same
way for janus_expert_ffn_vjp_split, and the library runs every GEMM of both
directions on kind::f16; the weights' FP16 splits for both directions are
written once per pass, in front of the forward (janus_expert_weights_f16, one
read of each weight tensor).  Below that size, re-splitting the weights every
call costs more than the FP16 GEMMs save, and the layer stays on 3xTF32.

`run_host` runs the pass from and to pinned host memory with the copies on
their own streams: the upload of G overlaps the forward, the download of Y
overlaps the VJP, and the next call's upload overlaps this call's compute
(inputs and outputs are double-buffered on the device).  When the input is
edge messages, they are streamed instead: the receivers are cut into chunks
whose messages fit a ring of device buffers, each chunk's messages are
uploaded into a free ring slot and aggregated from there as soon as they land,
so the messages never need a device copy of their own and the upload of the
next call's first chunks overlaps this call's MoE compute.
"""
import numpy as np
import torch

from . import janus as J


class MoELayer:
    OPS_FWD = ("route", "dispatch", "ffn_fwd", "combine")
    OPS_VJP = ("dispatch_w", "ffn_vjp", "combine_vjp")
    # this library's kernels per call (see each entry point's launches)
    LAUNCHES = {"edge_aggregate": 1, "quant": 2, "dequant": 1, "row_scales": 1, "route": 4, "dispatch": 1,
                "ffn_fwd": 2, "combine": 1, "dispatch_w": 1, "ffn_vjp": 2, "combine_vjp": 1}
    # the FP16 tensor path: row maxima + split dispatch; W1's split in front
    # of the two GEMMs
    LAUNCHES_SPLIT = {"dispatch": 2, "ffn_fwd": 3}
    SPLIT_MIN_ROWS_PER_EXPERT = None   # the library's rule (janus_expert_ffn_f16_min_rows_per_expert)

    # pinned-host pipeline for edge-message inputs: ring of device buffers
    RING_SLOTS = 8
    RING_SLOT_BYTES = 512 << 20

    def __init__(self, n_atoms, top_k, gate, w1, w2, *, mode=J.JANUS_FFN_3XTF32, packed=False,
                 row_ptr=None):
        """gate [T,E], w1 [E,d,h], w2 [E,h,d] on the layer's device.  packed:
        FP16 per-type packing of the dispatch.  row_ptr [N+1] (int64): the
        input is edge messages [Ed,d], aggregated per receiver first."""
        dev = w1.device
        self.dev = dev
        self.N, self.K = int(n_atoms), int(top_k)
        self.T, self.E = gate.shape
        _, self.d, self.h = w1.shape
        self.gate, self.w1, self.w2, self.mode = gate, w1, w2, mode
        self.packed, self.row_ptr = packed, row_ptr
        N, K, T, E, d, h = self.N, self.K, self.T, self.E, self.d, self.h
        R = N * K
        f32 = dict(dtype=torch.float32, device=dev)
        i32 = dict(dtype=torch.int32, device=dev)
        self.route_out = dict(topk_expert=torch.empty((N, K), **i32),
                              topk_weight=torch.empty((N, K), **f32),
                              counts=torch.empty((E,), **i32), offsets=torch.empty((E + 1,), **i32),
                              perm=torch.empty((R,), **i32), slot_of=torch.empty((R,), **i32))
        self.route_ws = torch.empty(J.janus_route_workspace_size(N, T, E, K), dtype=torch.uint8, device=dev)
        self.xd = torch.empty((R, d), **f32)
        self.yd = torch.empty((R, d), **f32)
        self.act = torch.empty((R, h), **f32)
        self.gd = torch.empty((R, d), **f32)
        self.dxd = torch.empty((R, d), **f32)
        self.y = torch.empty((N, d), **f32)
        self.dx = torch.empty((N, d), **f32)
        # packed: the first GEMM reads the FP16 payload itself (the unpack is
        # fused into it); its tensor-core form needs d % 8 == 0
        self.fused_unpack = packed and (mode == J.JANUS_FFN_FP32_SIMT or d % 8 == 0)
        # 3xTF32, unpacked rows: the forward's first GEMM on the FP16 tensor
        # path (rows split into two FP16 terms by the dispatch; d % 8 == 0)
        # when the rows per expert amortise the per-call weight split
        min_rows = (J.janus_expert_ffn_f16_min_rows_per_expert() if self.SPLIT_MIN_ROWS_PER_EXPERT is None
                    else self.SPLIT_MIN_ROWS_PER_EXPERT)
        self.split = (mode == J.JANUS_FFN_3XTF32 and not packed and d % 8 == 0
                      and R >= min_rows * E)
        # the input VJP on the FP16 tensor path (both GEMMs; the weighted
        # dispatch writes the gradient rows as two FP16 terms) on the same rule
        self.split_vjp = (mode == J.JANUS_FFN_3XTF32 and d % 8 == 0 and h % 8 == 0
                          and R >= min_rows * E)
        nb = max(J.janus_expert_ffn_workspace_size(R, d, h, E, False, True, mode),
                 J.janus_expert_ffn_workspace_size(R, d, h, E, True, True, mode),
                 J.janus_expert_ffn_packed_workspace_size(R, E, d, h, mode) if self.fused_unpack else 0,
                 J.janus_expert_ffn_split_workspace_size(R, E, d, h) if self.split or self.split_vjp else 0)
        self.ffn_ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        if self.split or self.split_vjp:
            self.split_ws = torch.empty(J.janus_dispatch_split_workspace_size(N), dtype=torch.uint8, device=dev)
        if self.split:
            self.xd16 = torch.empty((2 * R, d), dtype=torch.float16, device=dev)
            self.xd_scale = torch.empty((R,), **f32)
        if self.split_vjp:
            self.gd16 = torch.empty((2 * R, d), dtype=torch.float16, device=dev)
            self.gd_scale = torch.empty((R,), **f32)
        if row_ptr is not None:
            self.xagg = torch.empty((N, d), **f32)
        if packed:
            self.payload = torch.empty((R, d), dtype=torch.float16, device=dev)
            self.scale = torch.empty((T,), **f32)
            self.row_scale = torch.empty((R,), **f32)
            self.quant_ws = torch.empty(J.janus_quant_by_type_workspace_size(T), dtype=torch.uint8, device=dev)
        front = ("edge_aggregate",) if row_ptr is not None else ()
        if packed:
            mid = ("route", "quant", "row_scales" if self.fused_unpack else "dequant")
        else:
            mid = ("route", "dispatch")
        self.ops = front + mid + ("ffn_fwd", "combine") + self.OPS_VJP
        launches = dict(self.LAUNCHES)
        if self.split:
            launches.update(self.LAUNCHES_SPLIT)
        if self.packed and self.fused_unpack and mode == J.JANUS_FFN_3XTF32:
            launches["ffn_fwd"] = 3           # W1's split + the two GEMMs
        # the library also runs the forward's second GEMM on the FP16 path
        # (with H's row split and W2's split in front) from its row threshold
        # per expert with h % 8 == 0, after either FP16 first GEMM
        fp16_first = self.split or (self.packed and self.fused_unpack and mode == J.JANUS_FFN_3XTF32)
        self.f16_second = (fp16_first and h % 8 == 0
                           and R >= J.janus_expert_ffn_f16_min_rows_per_expert() * E)
        if self.f16_second:
            launches["ffn_fwd"] += 2          # H's row split + W2's split
        if self.split_vjp:
            # weighted split dispatch: row maxima + split; VJP: W2 split,
            # gd W2^T, dA's row split, W1 split, dA W1^T
            launches["dispatch_w"] = 2
            launches["ffn_vjp"] = 5
        # both directions on the FP16 path: the forward writes the splits of
        # both weight tensors for both directions (janus_expert_weights_f16,
        # one read of each tensor, 2 launches in place of the forward's two
        # splits) and the VJP launches none of its own
        self.w16set = None
        if self.f16_second and self.split_vjp:
            self.w16set = torch.empty(J.janus_expert_weights_f16_size(E, d, h), dtype=torch.uint8, device=dev)
            launches["ffn_vjp"] = 3
        self.launches_per_call = sum(launches[o] for o in self.ops)
        self._host = None

    # -- device-resident pass ----------------------------------------------------
    def forward_vjp(self, x, g, types, events=None, y=None, dx=None, after_forward=None, aggregated=False):
        """One pass on device tensors; returns (y, dx) (the layer's own buffers
        unless y / dx are given).  events: dict op -> (start, end) CUDA events;
        after_forward: called once y is enqueued, before the VJP; aggregated:
        the edge messages were already aggregated into self.xagg (x unused)."""
        K, T, r = self.K, self.T, self.route_out
        y = self.y if y is None else y
        dx = self.dx if dx is None else dx

        def mark(op, i):
            if events is not None:
                events[op][i].record()

        if aggregated:
            x = self.xagg
        elif self.row_ptr is not None:
            mark("edge_aggregate", 0)
            J.janus_edge_aggregate(x, self.row_ptr, out=self.xagg)
            mark("edge_aggregate", 1)
            x = self.xagg
        mark("route", 0)
        J.janus_route(types, self.gate, K, out=r, workspace=self.route_ws)
        mark("route", 1)
        if self.packed:
            mark("quant", 0)
            J.janus_quant_by_type(x, types, T, r["slot_of"], K, payload=self.payload, scale=self.scale,
                                  workspace=self.quant_ws)
            mark("quant", 1)
            if self.fused_unpack:
                mark("row_scales", 0)
                J.janus_dispatch_row_scales(types, T, r["perm"], K, self.scale, out=self.row_scale)
                mark("row_scales", 1)
            else:
                mark("dequant", 0)
                J.janus_dequant_by_type(self.payload, types, T, r["perm"], K, self.scale, out=self.xd)
                mark("dequant", 1)
        elif self.split:
            mark("dispatch", 0)
            J.janus_dispatch_split(x, r["slot_of"], K, out=self.xd16, row_scale=self.xd_scale, workspace=self.split_ws)
            mark("dispatch", 1)
        else:
            mark("dispatch", 0)
            J.janus_dispatch(x, r["slot_of"], K, out=self.xd)
            mark("dispatch", 1)
        mark("ffn_fwd", 0)
        if self.w16set is not None:
            J.janus_expert_weights_f16(self.w1, self.w2, J.JANUS_W16_FWD | J.JANUS_W16_VJP, out=self.w16set)
        if self.split:
            J.janus_expert_ffn_fwd_split(self.xd16, self.xd_scale, r["offsets"], self.w1, self.w2, out=self.yd,
                                         act=self.act, weights16=self.w16set, workspace=self.ffn_ws)
        elif self.fused_unpack:
            # the FP16 rows go straight into the first GEMM (xd is not written)
            J.janus_expert_ffn_fwd_packed(self.payload, self.row_scale, r["offsets"], self.w1, self.w2, out=self.yd,
                                          act=self.act, mode=self.mode, weights16=self.w16set,
                                          workspace=self.ffn_ws)
        else:
            # unpacked FP16 rows are exact in TF32: the first GEMM skips their residual
            J.janus_expert_ffn_fwd_ex(self.xd, r["offsets"], self.w1, self.w2, out=self.yd, act=self.act,
                                      flags=J.JANUS_FFN_X_DEQUANTIZED if self.packed else 0, mode=self.mode,
                                      workspace=self.ffn_ws)
        mark("ffn_fwd", 1)
        mark("combine", 0)
        J.janus_combine(self.yd, r["slot_of"], K, r["topk_weight"], out=y)
        mark("combine", 1)
        if after_forward is not None:
            after_forward()
        mark("dispatch_w", 0)
        if self.split_vjp:
            J.janus_dispatch_split(g, r["slot_of"], K, r["topk_weight"], out=self.gd16, row_scale=self.gd_scale,
                                   workspace=self.split_ws)
        else:
            J.janus_dispatch(g, r["slot_of"], K, r["topk_weight"], out=self.gd)
        mark("dispatch_w", 1)
        mark("ffn_vjp", 0)
        if self.split_vjp:
            J.janus_expert_ffn_vjp_split(self.gd16, self.gd_scale, r["offsets"], self.w1, self.w2, self.act,
                                         out=self.dxd, weights16=self.w16set, workspace=self.ffn_ws)
        else:
            # (xd is read only when the pre-activations are not saved; here they are)
            J.janus_expert_ffn_vjp(self.xd, self.gd, r["offsets"], self.w1, self.w2, act=self.act,
                                   mode=self.mode, out=self.dxd, workspace=self.ffn_ws)
        mark("ffn_vjp", 1)
        mark("combine_vjp", 0)
        J.janus_combine(self.dxd, r["slot_of"], K, out=dx)
        mark("combine_vjp", 1)
        return y, dx

    # -- pass from and to pinned host memory, copies overlapped -------------------
    def _edge_chunks(self, d):
        """Receiver chunks [i0, i1) whose messages [e0, e1) fit one ring slot,
        from the host copy of row_ptr (a receiver with more edges than a slot
        holds gets a chunk, and the slots that size, of its own)."""
        rp = self.row_ptr.cpu().numpy()
        slot_rows = max(1, self.RING_SLOT_BYTES // (4 * d))
        slot_rows = max(slot_rows, int((rp[1:] - rp[:-1]).max(initial=0)))
        chunks, i0 = [], 0
        N = rp.shape[0] - 1
        while i0 < N:
            # the last receiver i1 with rp[i1] - rp[i0] <= slot_rows
            i1 = int(np.searchsorted(rp, rp[i0] + slot_rows, side="right")) - 1
            i1 = max(i0 + 1, min(i1, N))
            chunks.append((i0, i1, int(rp[i0]), int(rp[i1])))
            i0 = i1
        return chunks, slot_rows

    def _host_state(self, x_shape):
        dev = self.dev
        f32 = dict(dtype=torch.float32, device=dev)
        st = {
            "copy_in": torch.cuda.Stream(dev), "copy_out": torch.cuda.Stream(dev), "k": 0,
            "g": [torch.empty((self.N, self.d), **f32) for _ in range(2)],
            "types": [torch.empty((self.N,), dtype=torch.int32, device=dev) for _ in range(2)],
            "y": [torch.empty((self.N, self.d), **f32) for _ in range(2)],
            "dx": [torch.empty((self.N, self.d), **f32) for _ in range(2)],
        }
        if self.row_ptr is None:
            st["x"] = [torch.empty(x_shape, **f32) for _ in range(2)]
        else:
            # edge messages: streamed through a ring of device buffers
            st["chunks"], slot_rows = self._edge_chunks(x_shape[1])
            n_slots = min(self.RING_SLOTS, max(1, len(st["chunks"])))
            st["ring"] = [torch.empty((slot_rows, x_shape[1]), **f32) for _ in range(n_slots)]
            st["ring_in"] = [torch.cuda.Event() for _ in range(n_slots)]
            st["ring_free"] = [torch.cuda.Event() for _ in range(n_slots)]
            st["ring_next"] = 0
            for ev in st["ring_free"]:
                ev.record(torch.cuda.current_stream(dev))
        for name in ("x_in", "g_in", "in_free", "y_done", "dx_done", "y_out", "dx_out"):
            st[name] = [torch.cuda.Event() for _ in range(2)]
        for b in range(2):      # nothing is in flight yet
            for name in ("in_free", "y_out", "dx_out"):
                st[name][b].record(torch.cuda.current_stream(dev))
        return st

    def _stream_edges(self, st, msg_h, s, cin):
        """Upload the edge messages chunk by chunk into the ring and aggregate
        each chunk into self.xagg on stream s as soon as it has landed."""
        ring = st["ring"]
        n = len(ring)
        for (i0, i1, e0, e1) in st["chunks"]:
            j = st["ring_next"] % n
            st["ring_next"] += 1
            cin.wait_event(st["ring_free"][j])
            with torch.cuda.stream(cin):
                ring[j][:e1 - e0].copy_(msg_h[e0:e1], non_blocking=True)
                st["ring_in"][j].record(cin)
            s.wait_event(st["ring_in"][j])
            J.janus_edge_aggregate(ring[j][:e1 - e0], self.row_ptr[i0:i1 + 1], out=self.xagg[i0:i1])
            st["ring_free"][j].record(s)

    def run_host(self, x_h, g_h, types_h, y_h, dx_h):
        """Enqueue one pass from pinned host inputs (x [N,d] or the edge
        messages [Ed,d], g [N,d], types [N]) into pinned host outputs y_h,
        dx_h.  Returns at once; the outputs are complete after `host_sync()`."""
        if self._host is None:
            self._host = self._host_state(tuple(x_h.shape))
        st = self._host
        b = st["k"] % 2
        st["k"] += 1
        s = torch.cuda.current_stream(self.dev)
        cin, cout = st["copy_in"], st["copy_out"]
        # inputs: buffer set b is free once the pass that last used it is done
        edges = self.row_ptr is not None
        cin.wait_event(st["in_free"][b])
        with torch.cuda.stream(cin):
            st["types"][b].copy_(types_h, non_blocking=True)
            if not edges:
                st["x"][b].copy_(x_h, non_blocking=True)
            st["x_in"][b].record(cin)
        s.wait_event(st["x_in"][b])
        if edges:
            self._stream_edges(st, x_h, s, cin)
        with torch.cuda.stream(cin):
            st["g"][b].copy_(g_h, non_blocking=True)
            st["g_in"][b].record(cin)
        s.wait_event(st["y_out"][b])           # y buffer b downloaded by its previous pass
        s.wait_event(st["dx_out"][b])

        def after_fwd():                        # y is final: download it during the VJP
            st["y_done"][b].record(s)
            cout.wait_event(st["y_done"][b])
            with torch.cuda.stream(cout):
                y_h.copy_(st["y"][b], non_blocking=True)
                st["y_out"][b].record(cout)
            s.wait_event(st["g_in"][b])

        self.forward_vjp(None if edges else st["x"][b], st["g"][b], st["types"][b], y=st["y"][b],
                         dx=st["dx"][b], after_forward=after_fwd, aggregated=edges)
        st["in_free"][b].record(s)
        st["dx_done"][b].record(s)
        cout.wait_event(st["dx_done"][b])
        with torch.cuda.stream(cout):
            dx_h.copy_(st["dx"][b], non_blocking=True)
            st["dx_out"][b].record(cout)

    def host_sync(self):
        """Make the current stream wait for every enqueued host pass's copies."""
        if self._host is not None:
            s = torch.cuda.current_stream(self.dev)
            for b in range(2):
                s.wait_event(self._host["y_out"][b])
                s.wait_event(self._host["dx_out"][b])
