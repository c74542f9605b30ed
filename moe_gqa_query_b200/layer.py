"""GQELayer: one GQE attention layer driven through the C ABI.

PyTorch supplies device memory (weights, activations, scratch) and the CUDA
stream; every step of the forward runs in libgqe.so's kernels:

  prefill  gqe_router_topk -> gqe_routed_qproj -> gqe_kv_proj ->
           gqe_attn_prefill -> gqe_combine_out_proj (output construction and
           projection, without materialising h where the shape allows)
  decode   gqe_router_topk -> gqe_routed_qproj -> gqe_kv_append ->
           gqe_attn_decode -> gqe_combine -> gqe_linear
  backward gqe_gemm (dh, dWo) -> gqe_combine_bwd -> gqe_attn_prefill_bwd ->
           gqe_router_bwd -> gqe_bwd_pack -> gqe_gemm (dx, dW_cat)

Weight layouts (bf16): Wr [D, G*E]; Wq [G, E, d, D]; Wk, Wv [G*d, D];
Wsh [n_shared*d, D]; Wo [D, slots*d] with slots = k*G + 1 + n_shared (GQE's
output; k*G + n_shared for the two ablation output modes).
"""
from __future__ import annotations

import dataclasses

import torch

from . import _lib as L


@dataclasses.dataclass(frozen=True)
class GQEConfig:
    B: int
    T: int
    D: int
    G: int
    E: int
    k: int
    d: int
    n_shared: int = 1
    sg: int = 0
    renorm_scope: int = 0
    scale: float = 0.0
    output_mode: int = 0

    @property
    def slots(self) -> int:
        return self.k * self.G + (1 if self.output_mode == 0 else 0) + self.n_shared


def config_from(obj) -> GQEConfig:
    return GQEConfig(**{f.name: getattr(obj, f.name) for f in dataclasses.fields(GQEConfig)
                        if hasattr(obj, f.name)})


class GQELayer:
    """Holds a layer's weights on one GPU and runs its forward passes."""

    def __init__(self, cfg, weights: dict, bias=None, device="cuda"):
        if not torch.cuda.is_available():
            raise RuntimeError("GQELayer needs a CUDA device; there is no CPU path")
        self.cfg = config_from(cfg)
        self.device = torch.device(device)
        c = self.cfg

        def dev(t, shape, dtype=torch.bfloat16):
            t = torch.as_tensor(t)
            if t.dtype == torch.int16 or t.dtype == torch.uint16:
                t = t.view(torch.bfloat16) if t.dtype == torch.int16 else t.view(torch.int16).view(torch.bfloat16)
            t = t.to(self.device, dtype).contiguous()
            if tuple(t.shape) != tuple(shape):
                raise ValueError(f"weight shape {tuple(t.shape)} != {tuple(shape)}")
            return t

        self.Wr = dev(weights["Wr"], (c.D, c.G * c.E))
        self.Wq = dev(weights["Wq"], (c.G, c.E, c.d, c.D))
        self.Wk = dev(weights["Wk"], (c.G * c.d, c.D))
        self.Wv = dev(weights["Wv"], (c.G * c.d, c.D))
        self.Wsh = dev(weights["Wsh"], (c.n_shared * c.d, c.D)) if c.n_shared else None
        self.Wo = dev(weights["Wo"], (c.D, c.slots * c.d))
        self.bias = None if bias is None else torch.as_tensor(bias, dtype=torch.float32).to(self.device).contiguous()
        self._bufs = {}
        self._graphs = {}
        self._side = None
        self.concurrent_kv = True

    # ------------------------------------------------------------------ buffers
    def _buf(self, name, shape, dtype=torch.bfloat16):
        t = self._bufs.get(name)
        if t is None or tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            t = torch.empty(shape, dtype=dtype, device=self.device)
            self._bufs[name] = t
        return t

    def _ws(self, name, nbytes):
        return self._buf(name, ((max(nbytes, 16) + 255) // 256 * 256,), torch.uint8)

    # ------------------------------------------------------------------ prefill
    def forward(self, x: torch.Tensor, stream=None, keep=False, out=None) -> torch.Tensor:
        """x [B, T, D] bf16 on the device -> y [B, T, D] bf16 (into `out` when given).

        keep=True also returns the intermediates (router outputs and probabilities,
        q, K, V, o, the log-sum-exp, h) that backward() reads.  They are the
        layer's own buffers: the next forward overwrites them, so run the
        backward of a step before the next step's forward.
        """
        c = self.cfg
        B, T = x.shape[0], x.shape[1]
        dims = L.make_dims(c, B=B, T=T)
        N = B * T
        idx = self._buf("idx", (N, c.G, c.k), torch.int32)
        w = self._buf("w", (N, c.G, c.k), torch.float32)
        q = self._buf("q", (B, c.G, T, c.k, c.d))
        qs = self._buf("qs", (B, T, c.d)) if c.n_shared else None
        K = self._buf("K", (B, c.G, T, c.d))
        V = self._buf("V", (B, c.G, T, c.d))
        o = self._buf("o", (B, c.G, T, c.k, c.d))
        os_ = self._buf("os", (B, T, c.d)) if c.n_shared else None
        y = self._buf("y", (B, T, c.D)) if out is None else out
        probs = self._buf("probs", (N, c.G, c.E), torch.float32) if keep else None
        lse = self._buf("lse", (N * c.G * c.k + N * c.n_shared,), torch.float32) if keep else None
        ws = self._ws("ws_q", L.gqe_workspace_size(dims, L.GQE_OP_ROUTED_QPROJ))
        ws_o = self._ws("ws_o", L.gqe_workspace_size(dims, L.GQE_OP_COMBINE_OUT_PROJ))
        if stream is None and self.concurrent_kv:
            # K/V depend on x alone: project them on a side stream while the
            # router, permutation and routed projection run (they leave SMs
            # idle in their ramps and tails); attention waits for both
            main = torch.cuda.current_stream(self.device)
            if self._side is None:
                self._side = torch.cuda.Stream(self.device)
            fork = torch.cuda.Event()
            fork.record(main)
            self._side.wait_event(fork)
            with torch.cuda.stream(self._side):
                L.gqe_kv_proj(dims, x, self.Wk, self.Wv, K, V)
                join = torch.cuda.Event()
                join.record(self._side)
            L.gqe_router_topk(dims, x, self.Wr, self.bias, idx, w, probs)
            L.gqe_routed_qproj(dims, x, self.Wq, self.Wsh, idx, q, qs, ws, None)
            main.wait_event(join)
        else:
            L.gqe_router_topk(dims, x, self.Wr, self.bias, idx, w, probs, stream)
            L.gqe_routed_qproj(dims, x, self.Wq, self.Wsh, idx, q, qs, ws, None, stream)
            L.gqe_kv_proj(dims, x, self.Wk, self.Wv, K, V, stream)
        L.gqe_attn_prefill(dims, q, qs, K, V, o, os_, lse, stream)
        L.gqe_combine_out_proj(dims, o, os_, w, self.Wo, y, ws_o, stream)
        if keep:
            h = self._buf("h", (N, c.slots * c.d))
            L.gqe_combine(dims, o, os_, w, h, stream)     # h itself, for the backward and inspection
            return y, dict(idx=idx, w=w, probs=probs, q=q, q_sh=qs, K=K, V=V, o=o, o_sh=os_, lse=lse, h=h)
        return y

    # ------------------------------------------------------------------ backward
    def backward(self, x: torch.Tensor, dy: torch.Tensor, saved: dict, stream=None) -> dict:
        """Gradients of <y, dy> for the forward(x, keep=True) that returned
        `saved`: dx [B, T, D] (bf16) and the fp32 weight gradients dWr, dbias,
        dWq, dWk, dWv, dWsh, dWo in the weights' layouts (summed over the
        tokens by split-K GEMMs with fp32 reduce-add).  TopK passes no gradient; the router learns
        through the weighted-sum slot (output_mode 0) or the weighted hard
        slots (mode 2).  The returned tensors are the layer's own buffers,
        overwritten by the next backward.

        The projection gradients go through one packed matrix A (gqe_bwd_pack):
        dx = A W_cat and dW_cat = A^T x with W_cat = [Wq; Wsh; Wk; Wv; Wr^T],
        where dq is scattered to its expert's columns (zeros for unselected
        experts, so the query part of these two GEMMs runs dense over all E
        experts of a group)."""
        c = self.cfg
        B, T = x.shape[0], x.shape[1]
        dims = L.make_dims(c, B=B, T=T)
        N, D, d, S = B * T, c.D, c.d, c.slots * c.d
        GE = c.G * c.E
        buf = self._buf
        # output projection: dh = dy Wo, dWo = dy^T h (operands read in place,
        # [K, M] / [K, N] layouts straight from memory)
        dy2 = dy.reshape(N, D)
        dh = buf("dh", (N, S))
        L.gqe_gemm(dy2, 0, self.Wo, 1, dh, stream)
        dWo = buf("dWo", (D, S), torch.float32)
        L.gqe_gemm_acc(dy2, 1, saved["h"], 1, dWo, False, stream)
        # output construction, attention, router
        do = buf("do", (B, c.G, T, c.k, d))
        do_sh = buf("do_sh", (B, T, d)) if c.n_shared else None
        dw = buf("dw", (N, c.G, c.k), torch.float32)
        L.gqe_combine_bwd(dims, saved["o"], saved["o_sh"], saved["w"], dh, do, do_sh, dw, stream)
        dq = buf("dq", (B, c.G, T, c.k, d))
        dq_sh = buf("dq_sh", (B, T, d)) if c.n_shared else None
        dK = buf("dK", (B, c.G, T, d))
        dV = buf("dV", (B, c.G, T, d))
        ws_a = self._ws("ws_a", L.gqe_workspace_size(dims, L.GQE_OP_ATTN_BWD))
        L.gqe_attn_prefill_bwd(dims, saved["q"], saved["q_sh"], saved["K"], saved["V"], saved["o"], saved["o_sh"],
                               saved["lse"], do, do_sh, dq, dq_sh, dK, dV, ws_a, stream)
        dlogits = buf("dlogits", (N, GE), torch.float32)
        dbias = buf("dbias", (GE,), torch.float32)
        L.gqe_router_bwd(dims, saved["probs"], saved["idx"], saved["w"], dw, dlogits, dbias, stream)
        # projections: dx = A W_cat, dW_cat = A^T x
        Kc = L.gqe_bwd_pack_cols(dims)
        Wcat = buf("Wcat", (Kc, D))
        L.gqe_bwd_pack_weights(dims, self.Wr, self.Wq, self.Wsh, self.Wk, self.Wv, Wcat, stream)
        A = buf("A", (N, Kc))
        L.gqe_bwd_pack(dims, saved["idx"], dq, dq_sh, dK, dV, dlogits, A, stream)
        dx = buf("dx", (B, T, D))
        L.gqe_gemm(A, 0, Wcat, 1, dx, stream)
        dWcat = buf("dWcat", (Kc, D), torch.float32)
        L.gqe_gemm_acc(A, 1, x.reshape(N, D), 1, dWcat, False, stream)
        r0 = GE * d
        r1 = r0 + c.n_shared * d
        r2 = r1 + c.G * d
        r3 = r2 + c.G * d
        dWr = buf("dWr", (D, GE), torch.float32)
        L.gqe_transpose_f32(dWcat[r3:r3 + GE], dWr, None, stream)
        return dict(dx=dx, dWr=dWr, dbias=dbias, dWq=dWcat[:r0].view(c.G, c.E, d, D),
                    dWsh=dWcat[r0:r1] if c.n_shared else None, dWk=dWcat[r1:r2], dWv=dWcat[r2:r3], dWo=dWo,
                    dh=dh, do=do, do_sh=do_sh, dw=dw, dq=dq, dq_sh=dq_sh, dK=dK, dV=dV, dlogits=dlogits)

    def forward_graph(self, x: torch.Tensor, out=None) -> torch.Tensor:
        """forward() replayed from a CUDA graph captured on first use for this
        input buffer, output buffer and shape (the six library calls become one
        graph launch), on the current stream.  Without `out` the returned tensor
        is the layer's own output buffer, overwritten by the next call."""
        key = (x.data_ptr(), tuple(x.shape), None if out is None else out.data_ptr())
        entry = self._graphs.get(key)
        if entry is None:
            self.forward(x, out=out)              # eager first: buffers, kernel attributes
            torch.cuda.synchronize(self.device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                y = self.forward(x, out=out)
            entry = self._graphs[key] = (g, y)
        g, y = entry
        g.replay()
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, graph: bool = True):
        """End-to-end call on host buffers (pinned for async copies): copy x in,
        run the forward (from a CUDA graph by default), copy y out, all on the
        current stream."""
        xd = self._buf("x_in", tuple(x_host.shape))
        xd.copy_(x_host, non_blocking=True)
        y = self.forward_graph(xd) if graph else self.forward(xd)
        y_host.copy_(y, non_blocking=True)
        return y_host

    def forward_host_c(self, x_host: torch.Tensor, y_host: torch.Tensor, chunk_seqs: int = 1, join: bool = True):
        """End to end in ONE C-ABI call, gqe_layer_forward_host: x_host [B, T, D]
        (pinned) -> y_host, the batch cut into chunks of chunk_seqs sequences
        whose copies in, forwards and copies back overlap on the layer's three
        streams, behind the current stream's work so far.  Returns an event
        that completes once y_host is written; with join=True the current
        stream also waits for it.  Calls in a row with join=False chain on the
        layer's streams, each call's copies overlapping the previous call's
        last steps; join once after the last one."""
        c = self.cfg
        B, T = x_host.shape[0], x_host.shape[1]
        chunk = max(1, int(chunk_seqs))
        # the scratch's layout depends on T and chunk_seqs alone, so batches of
        # any size chain on it; another layout gets another buffer (the old one
        # is released only after the streams' work on it, record_stream below)
        ws = self._ws("ws_host", L.gqe_workspace_size(L.make_dims(c, B=chunk, T=T), L.GQE_OP_LAYER_FORWARD_HOST))
        wstruct = L.layer_weights(self)     # read each call: the weight tensors may have been replaced
        cur = torch.cuda.current_stream(self.device)
        if getattr(self, "_pipe_streams", None) is None:
            self._pipe_streams = tuple(torch.cuda.Stream(self.device) for _ in range(3))
        s_in, s_cmp, s_out = self._pipe_streams
        start = torch.cuda.Event()
        start.record(cur)
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_event(start)
            ws.record_stream(s_)
        L.gqe_layer_forward_host(L.make_dims(c, B=B, T=T), wstruct, x_host, y_host, chunk, ws,
                                 s_in, s_cmp, s_out)
        done = torch.cuda.Event()
        done.record(s_cmp)          # the call leaves s_cmp behind its last copy back
        if join:
            cur.wait_event(done)
        return done

    def forward_host_pipelined(self, x_hosts, y_hosts):
        """End to end over a sequence of batches in (pinned) host memory:
        y_hosts[i] <- forward(x_hosts[i]).  The host->device copy of batch i,
        the forward of batch i-1 and the read-back of batch i-2 run at once on
        three streams over two device buffer sets, so the copies in the two
        directions overlap each other and the compute.  Everything is enqueued;
        the current stream waits for the last read-back, so synchronising it
        (or an event recorded on it) means every y_hosts[i] is written."""
        if len(x_hosts) != len(y_hosts):
            raise ValueError("x_hosts and y_hosts differ in length")
        if not x_hosts:
            return y_hosts
        cur = torch.cuda.current_stream(self.device)
        if getattr(self, "_pipe_streams", None) is None:
            self._pipe_streams = tuple(torch.cuda.Stream(self.device) for _ in range(3))
        s_in, s_cmp, s_out = self._pipe_streams
        B, T = x_hosts[0].shape[0], x_hosts[0].shape[1]
        xs = [self._buf(f"pipe_x{j}", (B, T, self.cfg.D)) for j in range(2)]
        ys = [self._buf(f"pipe_y{j}", (B, T, self.cfg.D)) for j in range(2)]
        start = torch.cuda.Event()
        start.record(cur)
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_event(start)
        done_cmp = [None, None]   # forward of the slot's last batch finished (x slot free)
        done_out = [None, None]   # read-back of the slot's last batch finished (y slot free)
        for i, (xh, yh) in enumerate(zip(x_hosts, y_hosts)):
            j = i & 1
            with torch.cuda.stream(s_in):
                if done_cmp[j] is not None:
                    s_in.wait_event(done_cmp[j])
                xs[j].copy_(xh, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ready)
                if done_out[j] is not None:
                    s_cmp.wait_event(done_out[j])
                self.forward_graph(xs[j], out=ys[j])
                done_cmp[j] = torch.cuda.Event()
                done_cmp[j].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_cmp[j])
                yh.copy_(ys[j], non_blocking=True)
                done_out[j] = torch.cuda.Event()
                done_out[j].record(s_out)
        for s_ in (s_in, s_cmp, s_out):
            cur.wait_stream(s_)
        return y_hosts

    # ------------------------------------------------------------------ decode
    def decode_step(self, x_new: torch.Tensor, Kc: torch.Tensor, Vc: torch.Tensor,
                    cache_len: torch.Tensor, stream=None, keep=False) -> torch.Tensor:
        """One new token per sequence.  x_new [B, D]; Kc, Vc [B, G, L_max, d]
        (the new token's K/V are written at row cache_len[b]-1); cache_len [B]
        int32 on the device.  Returns y [B, D]."""
        c = self.cfg
        B = x_new.shape[0]
        L_max = Kc.shape[2]
        dims = L.make_dims(c, B=B, T=1)
        idx = self._buf("d_idx", (B, c.G, c.k), torch.int32)
        w = self._buf("d_w", (B, c.G, c.k), torch.float32)
        q = self._buf("d_q", (B, c.G, 1, c.k, c.d))
        qs = self._buf("d_qs", (B, 1, c.d)) if c.n_shared else None
        o = self._buf("d_o", (B, c.G, 1, c.k, c.d))
        os_ = self._buf("d_os", (B, 1, c.d)) if c.n_shared else None
        h = self._buf("d_h", (B, c.slots * c.d))
        y = self._buf("d_y", (B, c.D))
        wsq = self._ws("d_ws_q", L.gqe_workspace_size(dims, L.GQE_OP_ROUTED_QPROJ))
        wsd = self._ws("d_ws_a", L.gqe_workspace_size(dims, L.GQE_OP_ATTN_DECODE, L_max))
        L.gqe_router_topk(dims, x_new, self.Wr, self.bias, idx, w, None, stream)
        L.gqe_routed_qproj(dims, x_new, self.Wq, self.Wsh, idx, q, qs, wsq, None, stream)
        L.gqe_kv_append(dims, x_new, self.Wk, self.Wv, Kc, Vc, L_max, cache_len, stream)
        L.gqe_attn_decode(dims, q, qs, Kc, Vc, L_max, cache_len, o, os_, wsd, stream)
        L.gqe_combine(dims, o, os_, w, h, stream)
        L.gqe_linear(h, self.Wo, y, stream)
        if keep:
            return y, dict(idx=idx, w=w, q=q, q_sh=qs, o=o, o_sh=os_, h=h)
        return y
