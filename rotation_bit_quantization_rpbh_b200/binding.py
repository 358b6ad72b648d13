"""Thin ctypes binding over liboq's C ABI (include/oq.h).

Argument marshalling only: every step of the path runs in liboq's kernels.
PyTorch supplies device memory and streams.  The calls keep the C names
without the ``oq_`` prefix.  Calls whose output buffers are omitted allocate
them with torch first (``quantize_acts(plan, cb, x)``).

If liboq.so is missing, the first call raises; there is no other
implementation behind these functions.
"""
import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboq.so")

OQ_OK = 0
OQ_BF16, OQ_F32 = 0, 1
OQ_ROT_RPBH, OQ_ROT_BLOCK_RHT = 0, 1
OQ_STARVE_RPBH, OQ_STARVE_GEMM = 1, 2
_STATUS = {0: "OQ_OK", 1: "OQ_ERR_INVALID_ARG", 2: "OQ_ERR_UNSUPPORTED", 3: "OQ_ERR_ALIGNMENT", 4: "OQ_ERR_CUDA",
           5: "OQ_ERR_TIMEOUT", 6: "OQ_ERR_OOM", 7: "OQ_ERR_NO_CONVERGENCE", 8: "OQ_ERR_TOO_LARGE"}
NOALLOC_SCRATCH_BYTES = 128 << 20

# every symbol include/oq.h declares
EXPORTS = ["oq_status_str", "oq_codebook", "oq_codebook_values", "oq_codebook_bf16", "oq_codebook_shape",
           "oq_codebook_free", "oq_rpbh_plan", "oq_rpbh_plan_export", "oq_rpbh_plan_host", "oq_rotation_plan",
           "oq_rotation_plan_host", "oq_plan_shape", "oq_qgemm_fp8", "oq_codebook_fp8",
           "oq_qlinear_fp8",
           "oq_plan_free", "oq_quantize_weights", "oq_quantize_acts", "oq_rpbh_apply", "oq_qgemm",
           "oq_qlinear_workspace", "oq_qlinear", "oq_qlinear_noalloc", "oq_device_status",
           "oq_debug_fail_allocations", "oq_debug_starve", "oq_quantize_acts_values",
           "oq_quantize_acts_values_fp8", "oq_qgemm_values", "oq_qgemm_values_fp8", "oq_qlinear_workspace_values",
           "oq_debug_rpbh_layout", "oq_codebook_upload", "oq_debug_qgemm_tile_rows",
           "oq_debug_rpbh_kernel"]


class OQError(RuntimeError):
    def __init__(self, status, call):
        self.status = status
        super().__init__(f"{call} failed: {_STATUS.get(status, status)}")


_lib = None
_lock = threading.Lock()


def lib():
    """Load liboq.so (fails loudly if it was not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"liboq.so not found at {LIB_PATH}; build it with "
                                       "`python -m rotation_bit_quantization_rpbh_b200.build`")
                L = ctypes.CDLL(LIB_PATH)
                P, I, U64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
                sig = {
                    "oq_status_str": ([I], ctypes.c_char_p),
                    "oq_codebook": ([I, I, P], I),
                    "oq_codebook_values": ([P, P, P], I),
                    "oq_codebook_bf16": ([P, P], I),
                    "oq_codebook_shape": ([P, P, P], I),
                    "oq_codebook_free": ([P], None),
                    "oq_codebook_upload": ([P], I),
                    "oq_rpbh_plan": ([I, I, U64, P], I),
                    "oq_rpbh_plan_export": ([P, P, P], I),
                    "oq_rpbh_plan_host": ([I, I, U64, P, P], I),
                    "oq_rotation_plan": ([I, I, U64, I, P], I),
                    "oq_rotation_plan_host": ([I, I, U64, I, P, P], I),
                    "oq_plan_shape": ([P, P, P], I),
                    "oq_plan_free": ([P], None),
                    "oq_quantize_weights": ([P, P, P, I, I, P, P, P], I),
                    "oq_quantize_acts": ([P, P, P, I, I, P, P, P], I),
                    "oq_rpbh_apply": ([P, P, I, I, P, P, P], I),
                    "oq_qgemm": ([P, P, I, I, P, P, P, P, P, P, P], I),
                    "oq_qgemm_fp8": ([P, P, I, I, P, P, P, P, P, P, P], I),
                    "oq_codebook_fp8": ([P, P], I),
                    "oq_qlinear_fp8": ([P, P, P, P, I, I, P, P, I, P, P, P, SZ, P], I),
                    "oq_qlinear_workspace": ([I, I, I], SZ),
                    "oq_qlinear": ([P, P, P, P, I, I, P, P, I, P, P, P, SZ, P], I),
                    "oq_qlinear_noalloc": ([P, P, P, P, I, I, P, P, I, P, P, P], I),
                    "oq_device_status": ([I, P, P], I),
                    "oq_debug_fail_allocations": ([I], None),
                    "oq_debug_starve": ([I], None),
                    "oq_debug_rpbh_layout": ([I, I, I], None),
                    "oq_debug_qgemm_tile_rows": ([I], None),
                    "oq_debug_rpbh_kernel": ([I], None),
                    "oq_quantize_acts_values": ([P, P, P, I, I, P, P, P], I),
                    "oq_quantize_acts_values_fp8": ([P, P, P, I, I, P, P, P], I),
                    "oq_qgemm_values": ([P, I, I, P, P, P, P, P, P, P], I),
                    "oq_qgemm_values_fp8": ([P, I, I, P, P, P, P, P, P, P], I),
                    "oq_qlinear_workspace_values": ([I, I], SZ),
                }
                for name, (args, res) in sig.items():
                    f = getattr(L, name)
                    f.argtypes = args
                    f.restype = res
                _lib = L
    return _lib


def _check(status, call):
    if status != OQ_OK:
        raise OQError(status, call)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return OQ_BF16
    if t.dtype == torch.float32:
        return OQ_F32
    raise TypeError(f"unsupported input dtype {t.dtype} (bf16 or fp32)")


def packed_row_bytes(d, bits):
    """Bytes of one packed row of d codes: one code per byte at 6 and 8 bits,
    else d * bits / 8 (3 bits: a bit stream, eight codes per three bytes)."""
    return d if bits in (6, 8) else d * bits // 8


def _need(t, name, shape, dtypes, device):
    """The C ABI sees only pointers and sizes: a tensor of the wrong shape,
    dtype, layout or device would make the kernels read or write out of
    bounds.  Check each buffer here and raise ValueError instead."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    if not isinstance(dtypes, tuple):
        dtypes = (dtypes,)
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _need_input(x, name, d):
    """x: a contiguous [rows, d] bf16 or fp32 CUDA tensor; returns rows."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{name} must be a 2-D torch.Tensor")
    if x.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    _need(x, name, (x.shape[0], d), (torch.bfloat16, torch.float32), x.device)
    return x.shape[0]


def _need_opt(t, name, shape, dtypes, device):
    if t is not None:
        _need(t, name, shape, dtypes, device)


class Codebook:
    """Lloyd-Max codebook C_d (library-owned handle)."""

    def __init__(self, d, bits):
        h = ctypes.c_void_p()
        _check(lib().oq_codebook(d, bits, ctypes.byref(h)), "oq_codebook")
        self._h = h
        self.d, self.bits, self.L = d, bits, 1 << bits

    @property
    def handle(self):
        return self._h

    def values(self):
        import numpy as np

        c = np.zeros(self.L)
        t = np.zeros(max(self.L - 1, 1))
        _check(lib().oq_codebook_values(self._h, c.ctypes.data_as(ctypes.c_void_p),
                                        t.ctypes.data_as(ctypes.c_void_p)), "oq_codebook_values")
        return c, t[: self.L - 1]

    def upload(self):
        """Put the quantiser tables on the current device now (set-up), so
        the quantising calls neither allocate nor synchronise later."""
        _check(lib().oq_codebook_upload(self._h), "oq_codebook_upload")
        return self

    def e4m3_bytes(self):
        """The fp8 variant's centroid values: e4m3 bytes of c_j sqrt(d)."""
        import numpy as np

        b = np.zeros(self.L, dtype=np.uint8)
        _check(lib().oq_codebook_fp8(self._h, b.ctypes.data_as(ctypes.c_void_p)), "oq_codebook_fp8")
        return b

    def bf16_bits(self):
        import numpy as np

        b = np.zeros(self.L, dtype=np.uint16)
        _check(lib().oq_codebook_bf16(self._h, b.ctypes.data_as(ctypes.c_void_p)), "oq_codebook_bf16")
        return b

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.oq_codebook_free(self._h)
            self._h = None


class Plan:
    """RPBH plan, or a rotation-ablation variant of it (library-owned handle
    with device tables on the current device)."""

    def __init__(self, d, h, seed, variant=OQ_ROT_RPBH):
        hp = ctypes.c_void_p()
        if variant == OQ_ROT_RPBH:
            _check(lib().oq_rpbh_plan(d, h, ctypes.c_uint64(seed), ctypes.byref(hp)), "oq_rpbh_plan")
        else:
            _check(lib().oq_rotation_plan(d, h, ctypes.c_uint64(seed), variant, ctypes.byref(hp)), "oq_rotation_plan")
        self._h = hp
        self.d, self.h, self.seed, self.variant = d, h, seed, variant

    @property
    def handle(self):
        return self._h

    def export(self):
        import numpy as np

        perm = np.zeros(self.d, dtype=np.int32)
        sign = np.zeros(self.d, dtype=np.int8)
        _check(lib().oq_rpbh_plan_export(self._h, perm.ctypes.data_as(ctypes.c_void_p),
                                         sign.ctypes.data_as(ctypes.c_void_p)), "oq_rpbh_plan_export")
        return perm, sign

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.oq_plan_free(self._h)
            self._h = None


def codebook(d, bits):
    return Codebook(d, bits)


def rpbh_plan(d, h, seed):
    return Plan(d, h, seed)


def rotation_plan(d, h, seed, variant):
    return Plan(d, h, seed, variant)


def rotation_plan_host(d, h, seed, variant):
    import numpy as np

    perm = np.zeros(d, dtype=np.int32)
    sign = np.zeros(d, dtype=np.int8)
    _check(lib().oq_rotation_plan_host(d, h, ctypes.c_uint64(seed), variant, perm.ctypes.data_as(ctypes.c_void_p),
                                       sign.ctypes.data_as(ctypes.c_void_p)), "oq_rotation_plan_host")
    return perm, sign


def rpbh_plan_host(d, h, seed):
    import numpy as np

    perm = np.zeros(d, dtype=np.int32)
    sign = np.zeros(d, dtype=np.int8)
    _check(lib().oq_rpbh_plan_host(d, h, ctypes.c_uint64(seed), perm.ctypes.data_as(ctypes.c_void_p),
                                   sign.ctypes.data_as(ctypes.c_void_p)), "oq_rpbh_plan_host")
    return perm, sign


def quantize_weights(plan, cb_w, W, idx_out=None, r_out=None, stream=None):
    N = _need_input(W, "W", plan.d)
    d = plan.d
    if idx_out is None:
        idx_out = torch.empty((N, packed_row_bytes(d, cb_w.bits)), dtype=torch.uint8, device=W.device)
    if r_out is None:
        r_out = torch.empty(N, dtype=torch.bfloat16, device=W.device)
    _need(idx_out, "idx_out", (N, packed_row_bytes(d, cb_w.bits)), torch.uint8, W.device)
    _need(r_out, "r_out", (N,), torch.bfloat16, W.device)
    _check(lib().oq_quantize_weights(plan.handle, cb_w.handle, _ptr(W), _dtype_code(W), N, _ptr(idx_out),
                                     _ptr(r_out), _stream(stream)), "oq_quantize_weights")
    return idx_out, r_out


def quantize_acts(plan, cb_a, x, idx_out=None, s_out=None, stream=None):
    M = _need_input(x, "x", plan.d)
    d = plan.d
    if idx_out is None:
        idx_out = torch.empty((M, packed_row_bytes(d, cb_a.bits)), dtype=torch.uint8, device=x.device)
    if s_out is None:
        s_out = torch.empty(M, dtype=torch.float32, device=x.device)
    _need(idx_out, "idx_out", (M, packed_row_bytes(d, cb_a.bits)), torch.uint8, x.device)
    _need(s_out, "s_out", (M,), torch.float32, x.device)
    _check(lib().oq_quantize_acts(plan.handle, cb_a.handle, _ptr(x), _dtype_code(x), M, _ptr(idx_out), _ptr(s_out),
                                  _stream(stream)), "oq_quantize_acts")
    return idx_out, s_out


def quantize_acts_values(plan, cb_a, x, val_out=None, s_out=None, stream=None, fp8=False):
    """The online pass writing the centroid values C_a[idx] (a bf16 tensor
    [M, d]) instead of the codes; ``fp8=True`` writes the e4m3 bytes of
    c sqrt(d) (uint8)."""
    M = _need_input(x, "x", plan.d)
    d = plan.d
    if val_out is None:
        val_out = torch.empty((M, d), dtype=torch.uint8 if fp8 else torch.bfloat16, device=x.device)
    if s_out is None:
        s_out = torch.empty(M, dtype=torch.float32, device=x.device)
    _need(val_out, "val_out", (M, d), torch.uint8 if fp8 else torch.bfloat16, x.device)
    _need(s_out, "s_out", (M,), torch.float32, x.device)
    fn, name = ((lib().oq_quantize_acts_values_fp8, "oq_quantize_acts_values_fp8") if fp8
                else (lib().oq_quantize_acts_values, "oq_quantize_acts_values"))
    _check(fn(plan.handle, cb_a.handle, _ptr(x), _dtype_code(x), M, _ptr(val_out), _ptr(s_out), _stream(stream)), name)
    return val_out, s_out


def rpbh_apply(plan, x, x_rot=None, norm_out=None, stream=None):
    M = _need_input(x, "x", plan.d)
    d = plan.d
    if x_rot is None:
        x_rot = torch.empty((M, d), dtype=torch.float32, device=x.device)
    if norm_out is None:
        norm_out = torch.empty(M, dtype=torch.float32, device=x.device)
    _need(x_rot, "x_rot", (M, d), torch.float32, x.device)
    _need(norm_out, "norm_out", (M,), torch.float32, x.device)
    _check(lib().oq_rpbh_apply(plan.handle, _ptr(x), _dtype_code(x), M, _ptr(x_rot), _ptr(norm_out),
                               _stream(stream)), "oq_rpbh_apply")
    return x_rot, norm_out


def _need_product(cb_w, a, a_name, a_cols, a_dtype, s, w_idx, w_r, bias, y):
    """Shapes of the product's buffers: a [M, a_cols], s [M] fp32, w_idx
    [N, packed row of cb_w], w_r [N] bf16, bias [N] bf16 or None, y [M, N]
    bf16 (allocated if None), all on a's CUDA device.  Returns (M, N, y)."""
    if not isinstance(a, torch.Tensor) or a.dim() != 2 or a.device.type != "cuda":
        raise ValueError(f"{a_name} must be a 2-D CUDA tensor")
    if not isinstance(w_idx, torch.Tensor) or w_idx.dim() != 2:
        raise ValueError("w_idx must be a 2-D tensor")
    M, N, dev = a.shape[0], w_idx.shape[0], a.device
    _need(a, a_name, (M, a_cols), a_dtype, dev)
    _need(s, "s", (M,), torch.float32, dev)
    _need(w_idx, "w_idx", (N, packed_row_bytes(cb_w.d, cb_w.bits)), torch.uint8, dev)
    _need(w_r, "w_r", (N,), torch.bfloat16, dev)
    _need_opt(bias, "bias", (N,), torch.bfloat16, dev)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _need(y, "y", (M, N), torch.bfloat16, dev)
    return M, N, y


def qgemm(cb_a, cb_w, a_idx, s, w_idx, w_r, bias=None, y=None, stream=None):
    M, N, y = _need_product(cb_w, a_idx, "a_idx", packed_row_bytes(cb_a.d, cb_a.bits), torch.uint8, s,
                            w_idx, w_r, bias, y)
    _check(lib().oq_qgemm(cb_a.handle, cb_w.handle, M, N, _ptr(a_idx), _ptr(s), _ptr(w_idx), _ptr(w_r), _ptr(bias),
                          _ptr(y), _stream(stream)), "oq_qgemm")
    return y


def qgemm_fp8(cb_a, cb_w, a_idx, s, w_idx, w_r, bias=None, y=None, stream=None):
    """oq_qgemm with e4m3 centroid values on the fp8 tensor cores."""
    M, N, y = _need_product(cb_w, a_idx, "a_idx", packed_row_bytes(cb_a.d, cb_a.bits), torch.uint8, s,
                            w_idx, w_r, bias, y)
    _check(lib().oq_qgemm_fp8(cb_a.handle, cb_w.handle, M, N, _ptr(a_idx), _ptr(s), _ptr(w_idx), _ptr(w_r),
                              _ptr(bias), _ptr(y), _stream(stream)), "oq_qgemm_fp8")
    return y


def qgemm_values(cb_w, a_val, s, w_idx, w_r, bias=None, y=None, stream=None, fp8=False):
    """The product with A given as centroid values (bf16 [M, d], or uint8
    e4m3 bytes with ``fp8=True``): only W is decoded in the kernel."""
    M, N, y = _need_product(cb_w, a_val, "a_val", cb_w.d, torch.uint8 if fp8 else torch.bfloat16, s, w_idx, w_r,
                            bias, y)
    fn, name = (lib().oq_qgemm_values_fp8, "oq_qgemm_values_fp8") if fp8 else (lib().oq_qgemm_values,
                                                                                "oq_qgemm_values")
    _check(fn(cb_w.handle, M, N, _ptr(a_val), _ptr(s), _ptr(w_idx), _ptr(w_r), _ptr(bias), _ptr(y), _stream(stream)),
           name)
    return y


def qlinear_workspace(M, d, bits_a):
    return int(lib().oq_qlinear_workspace(M, d, bits_a))


def qlinear_workspace_values(M, d):
    return int(lib().oq_qlinear_workspace_values(M, d))


def _need_layer(plan, cb_w, x, w_idx, w_r, bias, y, alloc_y):
    """The layer's buffers: x [M, plan d] bf16/fp32, w_idx [N, packed row of
    cb_w], w_r [N] bf16, bias [N] bf16 or None, y [M, N] bf16 (allocated
    here if None and alloc_y).  Returns (M, N, y, d)."""
    d = plan.d
    M = _need_input(x, "x", d)
    if not isinstance(w_idx, torch.Tensor) or w_idx.dim() != 2:
        raise ValueError("w_idx must be a 2-D tensor")
    N = w_idx.shape[0]
    _need(w_idx, "w_idx", (N, packed_row_bytes(d, cb_w.bits)), torch.uint8, x.device)
    _need(w_r, "w_r", (N,), torch.bfloat16, x.device)
    _need_opt(bias, "bias", (N,), torch.bfloat16, x.device)
    if y is None and alloc_y:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, "y", (M, N), torch.bfloat16, x.device)
    return M, N, y, d


def qlinear(plan, cb_a, cb_w, x, w_idx, w_r, bias=None, y=None, workspace=None, stream=None, fp8=False,
            schedule="auto"):
    """The full layer x -> y (oq_qlinear; oq_qlinear_fp8 with fp8=True).
    ``schedule`` sizes the workspace allocated here: "auto" (room for the
    values schedule, which the library then takes) or "codes"."""
    M, N, y, d = _need_layer(plan, cb_w, x, w_idx, w_r, bias, y, alloc_y=True)
    if schedule not in ("auto", "codes"):
        raise ValueError(f"unknown schedule {schedule!r}")
    if schedule == "auto":
        need = max(qlinear_workspace_values(M, d), qlinear_workspace(M, d, cb_a.bits))
    else:
        need = qlinear_workspace(M, d, cb_a.bits)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    if (not isinstance(workspace, torch.Tensor) or workspace.dtype != torch.uint8 or not workspace.is_contiguous()
            or workspace.device != x.device):
        raise ValueError("workspace must be a contiguous uint8 tensor on x's device")
    fn, name = (lib().oq_qlinear_fp8, "oq_qlinear_fp8") if fp8 else (lib().oq_qlinear, "oq_qlinear")
    _check(fn(plan.handle, cb_a.handle, cb_w.handle, _ptr(x), _dtype_code(x), M, _ptr(w_idx), _ptr(w_r), N,
              _ptr(bias), _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream)), name)
    return y


def qlinear_noalloc(plan, cb_a, cb_w, x, w_idx, w_r, y, bias=None, stream=None):
    """oq_qlinear without any device allocation inside the call, for callers
    that may not allocate device memory on their request path (a serving
    process that reserved all device memory at start-up).  The caller passes
    the output ``y``; the activations' values (or, if they do not fit, their
    packed codes) go to the library's fixed 128 MiB per-device scratch array,
    shared by all calls: calls that overlap on the GPU race on it, so keep
    them on one stream."""
    M, N, y, _ = _need_layer(plan, cb_w, x, w_idx, w_r, bias, y, alloc_y=False)
    _check(lib().oq_qlinear_noalloc(plan.handle, cb_a.handle, cb_w.handle, _ptr(x), _dtype_code(x), M, _ptr(w_idx),
                                    _ptr(w_r), N, _ptr(bias), _ptr(y), _stream(stream)), "oq_qlinear_noalloc")
    return y


def device_status(clear=True, stream=None):
    out = ctypes.c_int(0)
    _check(lib().oq_device_status(int(clear), ctypes.byref(out), _stream(stream)), "oq_device_status")
    return out.value


def debug_fail_allocations(n):
    """Test hook: the library's next ``n`` own device allocations fail
    (the calls making them return OQ_ERR_OOM); ``n <= 0`` cancels."""
    lib().oq_debug_fail_allocations(int(n))


def debug_starve(mask):
    """Test hook: the next launch of each kernel in ``mask``
    (OQ_STARVE_RPBH | OQ_STARVE_GEMM) issues no input copies, so its bounded
    waits run out and ``device_status()`` reports OQ_ERR_TIMEOUT.  Replaces
    the pending set; 0 cancels."""
    lib().oq_debug_starve(int(mask))


def debug_rpbh_layout(rows_per_warp=0, slots=0, lanes_per_block=0):
    """Test and tuning hook: force the team kernel's rows per
    warp (1, 2, 4, 8), staging slots per warp team (1, 2) and lanes per
    h-block (2: two lanes share a block; bf16 inputs, h of 64 or 128) where
    they fit; 0 restores the library's choice."""
    lib().oq_debug_rpbh_layout(int(rows_per_warp), int(slots), int(lanes_per_block))


def debug_qgemm_tile_rows(rows=0):
    """Test and tuning hook: tiles of 256 or 512 rows of A in the A-values
    product (0: the default, 256)."""
    lib().oq_debug_qgemm_tile_rows(int(rows))


RPBH_KERNEL_AUTO, RPBH_KERNEL_GROUPS, RPBH_KERNEL_TEAMS = 0, 1, 2


def debug_rpbh_kernel(which=RPBH_KERNEL_AUTO):
    """Test and tuning hook: the rotate-and-quantise kernel family for
    h <= 128 (1: warp groups, 2: teams; 0: the library's choice per shape)."""
    lib().oq_debug_rpbh_kernel(int(which))


def unpack_indices(packed, d, bits):
    """Unpack LSB-first packed indices [rows, bytes] to one index per byte
    [rows, d] (a layout conversion for tests and callers, on any device).
    3-bit codes are a bit stream, 8 codes per 3 bytes."""
    p = packed.to(torch.int32)
    if bits == 6:
        return (p & 63).to(torch.uint8)
    if bits == 3:
        rows = p.shape[0]
        b = p.reshape(rows, -1, 3)
        g = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)  # 24 bits = 8 codes
        shifts = torch.arange(8, device=p.device, dtype=torch.int32) * 3
        return ((g.unsqueeze(-1) >> shifts) & 7).reshape(rows, -1)[:, :d].to(torch.uint8)
    per = 8 // bits
    shifts = torch.arange(per, device=p.device, dtype=torch.int32) * bits
    v = (p.unsqueeze(-1) >> shifts) & ((1 << bits) - 1)
    return v.reshape(p.shape[0], -1)[:, :d].to(torch.uint8)
