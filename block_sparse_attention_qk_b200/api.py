"""Python binding of the C ABI (include/sbattn.h) for torch tensors.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels, on the current torch stream.  torch provides device memory and
streams.  Tensors must be CUDA, contiguous, [B, N, H, 128] bfloat16 (index
tensors int32).
"""

from __future__ import annotations

import ctypes

import torch

from ._lib import lib, strerror

BLOCK = 64
HEAD_DIM = 128


class SBAttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {strerror(code)} (status {code})")
        self.code = code


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn: str, rc: int):
    if rc != 0:
        raise SBAttnError(fn, rc)


def _act(name, t, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def check_status(status=None, device=None) -> None:
    """Synchronise the current stream and raise SBAttnError if a CUDA error
    surfaced or a kernel stored an error code in `status` (an int32 CUDA
    tensor of one element, as passed to `forward`)."""
    if status is not None:
        _act("status", status, torch.int32)
        device = status.device
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check("sbattn_check_status", lib().sbattn_check_status(_ptr(status), _stream(dev)))


def nblocks(N: int) -> int:
    return -(-N // BLOCK)


def keep_count(nblk: int, sparsity: float) -> int:
    """Kept key blocks per query block, diagonal included (host only)."""
    out = ctypes.c_int(0)
    _check("sbattn_keep_count", lib().sbattn_keep_count(int(nblk), float(sparsity), ctypes.byref(out)))
    return out.value


def qk_norm_rope(q, k, w_q, w_k, grid, *, dims=(32, 48, 48), theta=10000.0, eps=1e-6,
                 q_out=None, k_out=None, pool=False):
    """Fused QK-RMSNorm + 3D RoPE.  grid = (T, Hh, W) with N = T*Hh*W.

    Returns (q_rot, k_rot) or, with pool=True, (q_rot, k_rot, q_bar, k_bar)
    where the last two are the fp32 [B, H, nblk, d] block means."""
    _act("q", q), _act("k", k), _act("w_q", w_q), _act("w_k", w_k)
    B, N, H, d = q.shape
    T, Hh, W = grid
    q_out = torch.empty_like(q) if q_out is None else _act("q_out", q_out)
    k_out = torch.empty_like(k) if k_out is None else _act("k_out", k_out)
    q_bar = k_bar = None
    if pool:
        q_bar = torch.empty((B, H, nblocks(N), d), device=q.device, dtype=torch.float32)
        k_bar = torch.empty_like(q_bar)
    rc = lib().sbattn_qk_norm_rope(_ptr(q), _ptr(k), _ptr(w_q), _ptr(w_k), _ptr(q_out), _ptr(k_out),
                                   _ptr(q_bar), _ptr(k_bar), B, T, Hh, W, H, d, dims[0], dims[1], dims[2],
                                   float(theta), float(eps), _stream(q.device))
    _check("sbattn_qk_norm_rope", rc)
    return (q_out, k_out, q_bar, k_bar) if pool else (q_out, k_out)


def select_workspace_bytes(B, N, H, d=HEAD_DIM) -> int:
    return lib().sbattn_select_workspace_bytes(B, N, H, d)


def _select_outputs(B, H, nblk, cap, device, want_scores):
    kept_idx = torch.empty((B, H, nblk, cap), device=device, dtype=torch.int32)
    kept_cnt = torch.empty((B, H, nblk), device=device, dtype=torch.int32)
    scores = torch.empty((B, H, nblk, nblk), device=device, dtype=torch.float32) if want_scores else None
    return kept_idx, kept_cnt, scores


def select_blocks(q_rot, k_rot, sparsity, *, return_scores=False, workspace=None, capacity=None):
    """SubBlock selection (budget form) from rotated Q/K.
    Returns (kept_idx [B,H,nblk,K], kept_cnt [B,H,nblk]) (+ scores)."""
    _act("q_rot", q_rot), _act("k_rot", k_rot)
    B, N, H, d = q_rot.shape
    nblk = nblocks(N)
    K = keep_count(nblk, sparsity)
    cap = K if capacity is None else capacity
    kept_idx, kept_cnt, scores = _select_outputs(B, H, nblk, cap, q_rot.device, return_scores)
    need = select_workspace_bytes(B, N, H, d)
    if workspace is None:
        workspace = torch.empty(need, device=q_rot.device, dtype=torch.uint8)
    rc = lib().sbattn_select_blocks(_ptr(q_rot), _ptr(k_rot), B, N, H, d, float(sparsity), _ptr(kept_idx),
                                    _ptr(kept_cnt), cap, _ptr(scores), _ptr(workspace), workspace.numel(),
                                    _stream(q_rot.device))
    _check("sbattn_select_blocks", rc)
    return (kept_idx, kept_cnt, scores) if return_scores else (kept_idx, kept_cnt)


def select_blocks_noalloc(q_rot, k_rot, sparsity, *, return_scores=False, capacity=None):
    """select_blocks without a workspace: the pooled means use the library's
    built-in scratch array (for callers that cannot allocate device memory;
    limited to B * H * nblk <= 4096; calls that overlap on the GPU race)."""
    _act("q_rot", q_rot), _act("k_rot", k_rot)
    B, N, H, d = q_rot.shape
    nblk = nblocks(N)
    K = keep_count(nblk, sparsity)
    cap = K if capacity is None else capacity
    kept_idx, kept_cnt, scores = _select_outputs(B, H, nblk, cap, q_rot.device, return_scores)
    rc = lib().sbattn_select_blocks_noalloc(_ptr(q_rot), _ptr(k_rot), B, N, H, d, float(sparsity), _ptr(kept_idx),
                                            _ptr(kept_cnt), cap, _ptr(scores), _stream(q_rot.device))
    _check("sbattn_select_blocks_noalloc", rc)
    return (kept_idx, kept_cnt, scores) if return_scores else (kept_idx, kept_cnt)


def select_blocks_pooled(q_bar, k_bar, sparsity, *, return_scores=False, capacity=None):
    """Budget selection from pooled fp32 [B, H, nblk, d] block means."""
    _act("q_bar", q_bar, torch.float32), _act("k_bar", k_bar, torch.float32)
    B, H, nblk, d = q_bar.shape
    K = keep_count(nblk, sparsity)
    cap = K if capacity is None else capacity
    kept_idx, kept_cnt, scores = _select_outputs(B, H, nblk, cap, q_bar.device, return_scores)
    rc = lib().sbattn_select_blocks_pooled(_ptr(q_bar), _ptr(k_bar), B, nblk, H, d, float(sparsity),
                                           _ptr(kept_idx), _ptr(kept_cnt), cap, _ptr(scores),
                                           _stream(q_bar.device))
    _check("sbattn_select_blocks_pooled", rc)
    return (kept_idx, kept_cnt, scores) if return_scores else (kept_idx, kept_cnt)


def select_blocks_threshold(q_bar, k_bar, tau, *, return_scores=False):
    """Threshold selection: the diagonal plus every block with score >= tau."""
    _act("q_bar", q_bar, torch.float32), _act("k_bar", k_bar, torch.float32)
    B, H, nblk, d = q_bar.shape
    kept_idx, kept_cnt, scores = _select_outputs(B, H, nblk, nblk, q_bar.device, return_scores)
    rc = lib().sbattn_select_blocks_threshold(_ptr(q_bar), _ptr(k_bar), B, nblk, H, d, float(tau),
                                              _ptr(kept_idx), _ptr(kept_cnt), nblk, _ptr(scores),
                                              _stream(q_bar.device))
    _check("sbattn_select_blocks_threshold", rc)
    return (kept_idx, kept_cnt, scores) if return_scores else (kept_idx, kept_cnt)


def forward(q_rot, k_rot, v, kept_idx, kept_cnt, *, scale=None, out=None, status=None):
    """Block-sparse attention over the kept key blocks; returns out [B,N,H,d] bf16.

    status: optional int32 CUDA tensor of one element; device-side errors are
    recorded there (it is not cleared by the call)."""
    _act("q_rot", q_rot), _act("k_rot", k_rot), _act("v", v)
    _act("kept_idx", kept_idx, torch.int32), _act("kept_cnt", kept_cnt, torch.int32)
    B, N, H, d = q_rot.shape
    out = torch.empty_like(q_rot) if out is None else _act("out", out)
    if status is not None:
        _act("status", status, torch.int32)
    rc = lib().sbattn_forward(_ptr(q_rot), _ptr(k_rot), _ptr(v), _ptr(kept_idx), _ptr(kept_cnt),
                              kept_idx.shape[-1], _ptr(out), B, N, H, d,
                              0.0 if scale is None else float(scale), _ptr(status), _stream(q_rot.device))
    _check("sbattn_forward", rc)
    return out


def adaln_modulate(x, shift, scale, *, eps=1e-6, out=None):
    """AdaLN of x [B, N, C] bf16 with per-sample shift, scale [B, C] bf16:
    LayerNorm (no affine) * (1 + scale) + shift; returns bf16 [B, N, C]."""
    _act("x", x), _act("shift", shift), _act("scale", scale)
    B, N, C = x.shape
    if tuple(shift.shape) != (B, C) or tuple(scale.shape) != (B, C):
        raise ValueError("shift and scale must be [B, C]")
    out = torch.empty_like(x) if out is None else _act("out", out)
    rc = lib().sbattn_adaln_modulate(_ptr(x), _ptr(shift), _ptr(scale), _ptr(out), B, N, C, float(eps),
                                     _stream(x.device))
    _check("sbattn_adaln_modulate", rc)
    return out


def swiglu(gate, up=None, *, out=None):
    """silu(gate) * up.  With up=None, gate is a fused [rows, 2F] projection
    output whose first F columns are the gate and the last F the up half.
    Returns bf16 [rows, F]."""
    if up is None:
        h = _act("gate_up", gate)
        rows, two_f = h.reshape(-1, h.shape[-1]).shape
        if two_f % 2:
            raise ValueError("the fused projection output needs an even last dimension")
        F, ld = two_f // 2, two_f
        g_ptr = h.data_ptr()
        u_ptr = g_ptr + F * h.element_size()
        lead = h.shape[:-1]
        dev = h.device
    else:
        _act("gate", gate), _act("up", up)
        if gate.shape != up.shape:
            raise ValueError("gate and up must have the same shape")
        F = gate.shape[-1]
        rows, ld = gate.numel() // F, F
        g_ptr, u_ptr = gate.data_ptr(), up.data_ptr()
        lead = gate.shape[:-1]
        dev = gate.device
    out = torch.empty(tuple(lead) + (F,), device=dev, dtype=torch.bfloat16) if out is None else _act("out", out)
    rc = lib().sbattn_swiglu(ctypes.c_void_p(g_ptr), ctypes.c_void_p(u_ptr), _ptr(out), rows, F, ld, _stream(dev))
    _check("sbattn_swiglu", rc)
    return out


class AttentionLayer:
    """The whole hot path of one attention layer with preallocated device
    buffers: prologue (with fused block pooling) -> selection -> attention.

    `run_device` takes tensors already on the GPU.  `__call__` also takes
    host tensors (pinned, for asynchronous copies): then each call copies its
    inputs in and its output back, pipelined over two input/output slots so
    that the host-to-device copy of call i + 1 and the device-to-host copy of
    call i - 1 run on their own streams while call i computes.  The output
    host tensor of a call is complete once `drain()` (or a device
    synchronisation) follows it.
    """

    def __init__(self, B, T, Hh, W, H, sparsity, *, device="cuda", dims=(32, 48, 48), theta=10000.0,
                 eps=1e-6, fused_pool=True):
        self.B, self.T, self.Hh, self.W, self.H = B, T, Hh, W, H
        self.N = T * Hh * W
        self.nblk = nblocks(self.N)
        self.sparsity, self.dims, self.theta, self.eps = sparsity, dims, theta, eps
        self.fused_pool = fused_pool
        self.K = keep_count(self.nblk, sparsity)
        dev = torch.device(device)
        self.dev = dev
        self.shape = (B, self.N, H, HEAD_DIM)
        self.q_rot = torch.empty(self.shape, device=dev, dtype=torch.bfloat16)
        self.k_rot = torch.empty_like(self.q_rot)
        self.out = torch.empty_like(self.q_rot)
        self.q_bar = torch.empty((B, H, self.nblk, HEAD_DIM), device=dev, dtype=torch.float32)
        self.k_bar = torch.empty_like(self.q_bar)
        self.kept_idx = torch.empty((B, H, self.nblk, self.K), device=dev, dtype=torch.int32)
        self.kept_cnt = torch.empty((B, H, self.nblk), device=dev, dtype=torch.int32)
        self.status = torch.zeros((1,), device=dev, dtype=torch.int32)
        self.workspace = None if fused_pool else torch.empty(
            select_workspace_bytes(B, self.N, H), device=dev, dtype=torch.uint8)
        self._slots = None  # device input/output slots of the host-buffer path (allocated on first use)
        self._calls = 0

    def run_device(self, q, k, v, w_q, w_k, events=None, out=None):
        """Run the path on device tensors already resident in HBM; returns the
        output (`out` if given, else the layer's own output buffer).

        events: optional 4 CUDA events, recorded on the launching stream
        before the prologue, before the selection, before the attention and
        after it (per-kernel device timing)."""
        L, s = lib(), _stream(self.dev)
        B, N, H, d = self.B, self.N, self.H, HEAD_DIM
        out = self.out if out is None else out
        if events is not None:
            events[0].record()
        if self.fused_pool:
            rc = L.sbattn_qk_norm_rope(_ptr(q), _ptr(k), _ptr(w_q), _ptr(w_k), _ptr(self.q_rot), _ptr(self.k_rot),
                                       _ptr(self.q_bar), _ptr(self.k_bar), B, self.T, self.Hh, self.W, H, d,
                                       *self.dims, float(self.theta), float(self.eps), s)
            _check("sbattn_qk_norm_rope", rc)
            if events is not None:
                events[1].record()
            rc = L.sbattn_select_blocks_pooled(_ptr(self.q_bar), _ptr(self.k_bar), B, self.nblk, H, d,
                                               float(self.sparsity), _ptr(self.kept_idx), _ptr(self.kept_cnt),
                                               self.K, None, s)
            _check("sbattn_select_blocks_pooled", rc)
        else:
            rc = L.sbattn_qk_norm_rope(_ptr(q), _ptr(k), _ptr(w_q), _ptr(w_k), _ptr(self.q_rot), _ptr(self.k_rot),
                                       None, None, B, self.T, self.Hh, self.W, H, d,
                                       *self.dims, float(self.theta), float(self.eps), s)
            _check("sbattn_qk_norm_rope", rc)
            if events is not None:
                events[1].record()
            rc = L.sbattn_select_blocks(_ptr(self.q_rot), _ptr(self.k_rot), B, N, H, d, float(self.sparsity),
                                        _ptr(self.kept_idx), _ptr(self.kept_cnt), self.K, None,
                                        _ptr(self.workspace), self.workspace.numel(), s)
            _check("sbattn_select_blocks", rc)
        if events is not None:
            events[2].record()
        rc = L.sbattn_forward(_ptr(self.q_rot), _ptr(self.k_rot), _ptr(v), _ptr(self.kept_idx),
                              _ptr(self.kept_cnt), self.K, _ptr(out), B, N, H, d, 0.0,
                              _ptr(self.status), s)
        _check("sbattn_forward", rc)
        if events is not None:
            events[3].record()
        return out

    # kernels launched per run_device call (prologue, selection [+ pooling], attention)
    @property
    def launches_per_call(self) -> int:
        return 3 if self.fused_pool else 4

    def _host_slots(self):
        if self._slots is None:
            mk = lambda shape: torch.empty(shape, device=self.dev, dtype=torch.bfloat16)
            self._slots = [dict(q=mk(self.shape), k=mk(self.shape), v=mk(self.shape), w_q=mk((HEAD_DIM,)),
                                w_k=mk((HEAD_DIM,)), out=mk(self.shape),
                                ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(), ev_out=torch.cuda.Event(),
                                used=False)
                           for _ in range(2)]
            self._h2d = torch.cuda.Stream(self.dev)
            self._d2h = torch.cuda.Stream(self.dev)
        return self._slots

    def __call__(self, q, k, v, w_q, w_k, out_host=None):
        if q.is_cuda:
            return self.run_device(q, k, v, w_q, w_k)
        slots = self._host_slots()
        sl = slots[self._calls % 2]
        comp = torch.cuda.current_stream(self.dev)
        with torch.cuda.stream(self._h2d):
            if sl["used"]:
                self._h2d.wait_event(sl["ev_done"])  # the slot's previous inputs have been consumed
            for name, src in (("q", q), ("k", k), ("v", v), ("w_q", w_q), ("w_k", w_k)):
                sl[name].copy_(src, non_blocking=True)
            sl["ev_in"].record(self._h2d)
        comp.wait_event(sl["ev_in"])
        if sl["used"]:
            comp.wait_event(sl["ev_out"])  # the slot's previous output has been read back
        o = self.run_device(sl["q"], sl["k"], sl["v"], sl["w_q"], sl["w_k"], out=sl["out"])
        sl["ev_done"].record(comp)
        if out_host is None:
            out_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        with torch.cuda.stream(self._d2h):
            self._d2h.wait_event(sl["ev_done"])
            out_host.copy_(o, non_blocking=True)
            sl["ev_out"].record(self._d2h)
        sl["used"] = True
        self._calls += 1
        return out_host

    def drain(self):
        """Make the current stream wait for every copy issued by host-buffer
        calls (events recorded on it afterwards include them)."""
        if self._slots is not None:
            comp = torch.cuda.current_stream(self.dev)
            comp.wait_stream(self._h2d)
            comp.wait_stream(self._d2h)

    def check_status(self):
        """Synchronise and raise if a kernel recorded a device-side error."""
        check_status(self.status)


def attention_flops(B, N, H, K, d=HEAD_DIM) -> float:
    """Effective FLOPs of the attention over the kept blocks: 4 * N * (64 K) * d
    per (batch, head) -- QK^T and PV at two flops per multiply-add, 64 keys per
    kept block."""
    return 4.0 * B * H * N * (BLOCK * K) * d
