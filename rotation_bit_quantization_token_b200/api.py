"""Python binding of libfq: the C ABI calls with torch tensors for device memory.

Every step of the operator runs in libfq's CUDA kernels; this module only checks
tensor placement, allocates outputs with torch, and passes pointers and the current
CUDA stream. There is no CPU implementation here.
"""

import ctypes

import torch

from . import _lib

_DT = {torch.bfloat16: _lib.FQ_BF16, torch.float16: _lib.FQ_FP16}


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check_input(name, t, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libfq has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")


def _check_device(x, **others):
    """x on the current CUDA device (the plan was made, and its kernels launch, there) and
    every other tensor beside it."""
    cur = torch.cuda.current_device()
    if x.device.index != cur:
        raise ValueError(f"x is on {x.device} but the current CUDA device is cuda:{cur}; "
                         "call torch.cuda.set_device first")
    for name, t in others.items():
        if t is not None and t.device != x.device:
            raise ValueError(f"{name} must be on {x.device}, got {t.device}")


def _check_output(name, t, nbytes, device, dtype=None):
    """A caller-supplied output: on `device`, contiguous, exactly `nbytes` bytes (the
    kernel writes all of them, so a smaller buffer would be overrun), and of `dtype` when
    the values are numbers rather than packed codes."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    have = t.numel() * t.element_size()
    if have != nbytes:
        raise ValueError(f"{name} must hold {nbytes} bytes, got {have}")


def _scale_bytes(K, M, N):
    return K * (-(-M * N // 64)) * 2


class FlatQuant:
    """A plan for one shape [K, M, N] and input dtype (the handle of fq_create)."""

    def __init__(self, K, M, N, dtype=torch.bfloat16, kernel="auto"):
        lib = _lib.load()
        if dtype not in _DT:
            raise ValueError("dtype must be torch.bfloat16 or torch.float16")
        self.K, self.M, self.N, self.dtype = int(K), int(M), int(N), dtype
        h = ctypes.c_void_p()
        _lib.check(lib.fq_create(ctypes.byref(h), self.K, self.M, self.N, _DT[dtype]),
                   "fq_create")
        self._h = h
        self._lib = lib
        self.set_kernel(kernel)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.fq_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_kernel(self, kernel):
        code = {"auto": _lib.FQ_KERNEL_AUTO, "general": _lib.FQ_KERNEL_GENERAL,
                "tcgen05": _lib.FQ_KERNEL_TCGEN05}[kernel]
        _lib.check(self._lib.fq_set_kernel(self._h, code), "fq_set_kernel")
        self.kernel = kernel

    def set_intermediate_rounding(self, enable):
        """Round x' = x . P2 to the input dtype before the left product (see
        fq_set_intermediate_rounding); runs the general kernel."""
        _lib.check(self._lib.fq_set_intermediate_rounding(self._h, int(bool(enable))),
                   "fq_set_intermediate_rounding")
        self.intermediate_rounding = bool(enable)

    def debug_arm_stall(self, wait_limit_s):
        """Test hook: the next tensor-core launch issues no x loads and every bounded wait in
        it gives up after wait_limit_s seconds (see fq_debug_arm_stall)."""
        _lib.check(self._lib.fq_debug_arm_stall(self._h, float(wait_limit_s)), "fq_debug_arm_stall")

    @property
    def last_kernel(self):
        return {0: "auto", 1: "general", 2: "tcgen05"}[self._lib.fq_last_kernel(self._h)]

    @property
    def last_launch_count(self):
        return self._lib.fq_last_launch_count(self._h)

    def device_status(self):
        v = ctypes.c_uint32(0)
        st = self._lib.fq_device_status(self._h, ctypes.byref(v))
        if st not in (_lib.FQ_OK, _lib.FQ_ERR_DEVICE_TIMEOUT):
            _lib.check(st, "fq_device_status")
        return int(v.value)

    def _inputs(self, x, P1, P2, allow_no_p2=False):
        _check_input("x", x, self.dtype)
        _check_input("P1", P1, self.dtype)
        if tuple(x.shape) != (self.K, self.M, self.N):
            raise ValueError(f"x must have shape {(self.K, self.M, self.N)}, got {tuple(x.shape)}")
        if tuple(P1.shape) != (self.M, self.M):
            raise ValueError("P1 must be [M, M]")
        if P2 is not None and P2.numel() == 0 and allow_no_p2:
            P2 = None
        if P2 is None:
            if not allow_no_p2:
                raise ValueError("P2 is required in per-token mode")
        else:
            _check_input("P2", P2, self.dtype)
            if tuple(P2.shape) != (self.N, self.N):
                raise ValueError("P2 must be [N, N]")
        _check_device(x, P1=P1, P2=P2)
        return P2

    def quantize_per_token(self, x, P1, P2, clip_ratio=1.0, out_dtype="int4",
                           out=None, quant_scale=None, stream=None):
        """Per-token INT4 quantization of P1 . (x . P2). Returns (out, quantScale):
        out is uint8 [K, M*N/2] for "int4" or int32 [K, M, N/8] for "int32"."""
        self._inputs(x, P1, P2)
        K, M, N = self.K, self.M, self.N
        if out is None:
            if out_dtype == "int32":
                out = torch.empty((K, M, N // 8), dtype=torch.int32, device=x.device)
            else:
                out = torch.empty((K, M * N // 2), dtype=torch.uint8, device=x.device)
        else:
            _check_output("out", out, K * M * N // 2, x.device)
        if quant_scale is None:
            quant_scale = torch.empty((K,), dtype=torch.float32, device=x.device)
        else:
            _check_output("quant_scale", quant_scale, 4 * K, x.device, torch.float32)
        fmt = _lib.FQ_OUT_INT32 if out_dtype == "int32" else _lib.FQ_OUT_INT4
        _lib.check(self._lib.fq_quantize_per_token(
            self._h, _ptr(x), _ptr(P1), _ptr(P2), float(clip_ratio), fmt, _ptr(out),
            _ptr(quant_scale), _stream_ptr(stream)), "fq_quantize_per_token")
        return out, quant_scale

    def quantize_mx(self, x, P1, P2, dst_type_max=0.0, out=None, scales=None, stream=None):
        """Per-group E2M1 + E8M0 quantization of P1 . (x . P2) (P2 None skips the right
        multiply). Returns (out uint8 [K, M*N/2], scales uint8 [K, ceilDiv(M*N,64), 2])."""
        P2 = self._inputs(x, P1, P2, allow_no_p2=True)
        K, M, N = self.K, self.M, self.N
        if out is None:
            out = torch.empty((K, M * N // 2), dtype=torch.uint8, device=x.device)
        else:
            _check_output("out", out, K * M * N // 2, x.device)
        if scales is None:
            scales = torch.empty((K, -(-M * N // 64), 2), dtype=torch.uint8, device=x.device)
        else:
            _check_output("scales", scales, _scale_bytes(K, M, N), x.device)
        _lib.check(self._lib.fq_quantize_mx(
            self._h, _ptr(x), _ptr(P1), _ptr(P2), float(dst_type_max), _ptr(out),
            _ptr(scales), _stream_ptr(stream)), "fq_quantize_mx")
        return out, scales

    def debug_rotate(self, x, P1, P2, out=None, stream=None):
        """x'' = P1 . (x . P2) as float32 [K, M, N] (test hook)."""
        P2 = self._inputs(x, P1, P2, allow_no_p2=True)
        if out is None:
            out = torch.empty((self.K, self.M, self.N), dtype=torch.float32, device=x.device)
        else:
            _check_output("out", out, 4 * self.K * self.M * self.N, x.device, torch.float32)
        _lib.check(self._lib.fq_debug_rotate(self._h, _ptr(x), _ptr(P1), _ptr(P2), _ptr(out),
                                             _stream_ptr(stream)), "fq_debug_rotate")
        return out


def quantize_per_token(x, P1, P2, clip_ratio=1.0, out_dtype="int4", kernel="auto"):
    K, M, N = x.shape
    return FlatQuant(K, M, N, x.dtype, kernel).quantize_per_token(x, P1, P2, clip_ratio, out_dtype)


def quantize_mx(x, P1, P2, dst_type_max=0.0, kernel="auto"):
    K, M, N = x.shape
    return FlatQuant(K, M, N, x.dtype, kernel).quantize_mx(x, P1, P2, dst_type_max)


def quantize_mx_static(x, P1, P2, dst_type_max=0.0, out=None, scales=None, stream=None):
    """Per-group quantization through fq_quantize_mx_static: no handle, and the library
    allocates nothing (its scratch is a static device array). Outputs are allocated here
    by torch unless passed in."""
    lib = _lib.load()
    if x.dtype not in _DT:
        raise ValueError("x must be bfloat16 or float16")
    for name, t in (("x", x), ("P1", P1)):
        _check_input(name, t, x.dtype)
    if P2 is not None and P2.numel() == 0:
        P2 = None
    if P2 is not None:
        _check_input("P2", P2, x.dtype)
    if x.dim() != 3:
        raise ValueError("x must be [K, M, N]")
    K, M, N = x.shape
    if tuple(P1.shape) != (M, M):
        raise ValueError("P1 must be [M, M]")
    if P2 is not None and tuple(P2.shape) != (N, N):
        raise ValueError("P2 must be [N, N]")
    _check_device(x, P1=P1, P2=P2)
    if out is None:
        out = torch.empty((K, M * N // 2), dtype=torch.uint8, device=x.device)
    else:
        _check_output("out", out, K * M * N // 2, x.device)
    if scales is None:
        scales = torch.empty((K, -(-M * N // 64), 2), dtype=torch.uint8, device=x.device)
    else:
        _check_output("scales", scales, _scale_bytes(K, M, N), x.device)
    _lib.check(lib.fq_quantize_mx_static(K, M, N, _DT[x.dtype], _ptr(x), _ptr(P1), _ptr(P2),
                                         float(dst_type_max), _ptr(out), _ptr(scales),
                                         _stream_ptr(stream)), "fq_quantize_mx_static")
    return out, scales


def debug_rotate(x, P1, P2, kernel="auto"):
    K, M, N = x.shape
    return FlatQuant(K, M, N, x.dtype, kernel).debug_rotate(x, P1, P2)


class HostPipeline:
    """End-to-end use from host memory. The tokens are processed in `chunks` equal slices:
    the host-to-device copy of slice c + 1, the operator on slice c and the device-to-host
    copy of slice c - 1 run on three streams at once (the copy engines work in both
    directions together), so a step costs about its larger transfer instead of the sum.
    Device buffers, streams and the per-slice handle are allocated once, in the
    constructor. With chunks = 1, or when K is not a multiple of `chunks`, everything runs
    on the caller's stream in one slice."""

    def __init__(self, fq: FlatQuant, mode, out_dtype="int4", device=None, chunks=8):
        self.fq = fq
        self.mode = mode
        self.out_dtype = out_dtype
        dev = device or torch.device("cuda", torch.cuda.current_device())
        K, M, N = fq.K, fq.M, fq.N
        self.x = torch.empty((K, M, N), dtype=fq.dtype, device=dev)
        self.P1 = torch.empty((M, M), dtype=fq.dtype, device=dev)
        self.P2 = torch.empty((N, N), dtype=fq.dtype, device=dev)
        if mode == "per_token":
            if out_dtype == "int32":
                self.out = torch.empty((K, M, N // 8), dtype=torch.int32, device=dev)
            else:
                self.out = torch.empty((K, M * N // 2), dtype=torch.uint8, device=dev)
            self.scale = torch.empty((K,), dtype=torch.float32, device=dev)
        else:
            self.out = torch.empty((K, M * N // 2), dtype=torch.uint8, device=dev)
            self.scale = torch.empty((K, -(-M * N // 64), 2), dtype=torch.uint8, device=dev)
        self.chunks = chunks if chunks >= 1 and K % chunks == 0 else 1
        self.kc = K // self.chunks
        if self.chunks > 1:
            self.fq_c = FlatQuant(self.kc, M, N, fq.dtype, kernel=getattr(fq, "kernel", "auto"))
            self.s_in = torch.cuda.Stream(dev)
            self.s_out = torch.cuda.Stream(dev)

    def host_outputs(self):
        """Pinned host buffers shaped like the outputs."""
        return (torch.empty_like(self.out, device="cpu").pin_memory(),
                torch.empty_like(self.scale, device="cpu").pin_memory())

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.x, self.P1, self.P2))

    def d2h_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.out, self.scale))

    def _launch(self, fq, x, out, scale, clip_ratio, dst_type_max, s):
        if self.mode == "per_token":
            fq.quantize_per_token(x, self.P1, self.P2, clip_ratio, self.out_dtype,
                                  out=out, quant_scale=scale, stream=s)
        else:
            fq.quantize_mx(x, self.P1, self.P2, dst_type_max, out=out, scales=scale, stream=s)

    def run(self, x_host, P1_host, P2_host, out_host, scale_host, clip_ratio=1.0,
            dst_type_max=0.0, stream=None):
        s = stream if stream is not None else torch.cuda.current_stream()
        if self.chunks == 1:
            with torch.cuda.stream(s):
                self.x.copy_(x_host, non_blocking=True)
                self.P1.copy_(P1_host, non_blocking=True)
                self.P2.copy_(P2_host, non_blocking=True)
                self._launch(self.fq, self.x, self.out, self.scale, clip_ratio, dst_type_max, s)
                out_host.copy_(self.out, non_blocking=True)
                scale_host.copy_(self.scale, non_blocking=True)
            return out_host, scale_host
        # the side streams start after everything queued on the caller's stream so far
        # (the previous step included), and the caller's stream ends after the last copy out
        start = torch.cuda.Event()
        start.record(s)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        with torch.cuda.stream(self.s_in):
            self.P1.copy_(P1_host, non_blocking=True)
            self.P2.copy_(P2_host, non_blocking=True)
        for c in range(self.chunks):
            sl = slice(c * self.kc, (c + 1) * self.kc)
            with torch.cuda.stream(self.s_in):
                self.x[sl].copy_(x_host[sl], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(self.s_in)
            s.wait_event(landed)
            with torch.cuda.stream(s):
                self._launch(self.fq_c, self.x[sl], self.out[sl], self.scale[sl], clip_ratio,
                             dst_type_max, s)
                done = torch.cuda.Event()
                done.record(s)
            self.s_out.wait_event(done)
            with torch.cuda.stream(self.s_out):
                out_host[sl].copy_(self.out[sl], non_blocking=True)
                scale_host[sl].copy_(self.scale[sl], non_blocking=True)
        end = torch.cuda.Event()
        end.record(self.s_out)
        s.wait_event(end)
        return out_host, scale_host
