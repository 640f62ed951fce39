"""ctypes binding of libhsnf4.so (the C ABI in include/hsnf4.h).

Argument marshalling only: torch tensors provide device memory and streams,
every step of the path runs in the library's CUDA kernels.  There is no
fallback -- if the library or a CUDA device is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_float, c_int, c_int64, c_size_t, c_uint32, \
    c_uint64, c_void_p
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhsnf4.so")
MAX_PROJ = 8

OK, ERR_INVALID, ERR_OOM, ERR_CUDA, ERR_TIMEOUT, ERR_STATE, ERR_DEVICE = range(7)
BASE_NF4, BASE_BF16 = 0, 1  # formats of the frozen base weight


class Nf4WeightC(Structure):
    _fields_ = [("codes", c_void_p), ("absmax", c_void_p), ("n_out", c_int64), ("k_in", c_int64),
                ("format", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_DROPOUT_FIELDS = [("dropout_p", c_float), ("reserved", ctypes.c_uint32),
                   ("dropout_seed", c_uint64), ("dropout_offset", c_uint64)]


class FwdArgs(Structure):
    _fields_ = [("W", Nf4WeightC), ("X", c_void_p), ("A", c_void_p), ("B", c_void_p),
                ("Y", c_void_p), ("t_save", c_void_p)] + _DROPOUT_FIELDS


class BwdArgs(Structure):
    _fields_ = [("W", Nf4WeightC), ("X", c_void_p), ("t_save", c_void_p), ("A", c_void_p),
                ("B", c_void_p), ("dY", c_void_p), ("dX", c_void_p), ("dA", c_void_p),
                ("dB", c_void_p)] + _DROPOUT_FIELDS


class LayerDesc(Structure):
    _fields_ = [("n_proj", c_int), ("n_out", c_int64 * MAX_PROJ), ("k_in", c_int64 * MAX_PROJ),
                ("base_format", c_int)]


# int gather(void *slot, size_t shard_bytes, int world, int block, void *copy_stream, void *user)
GATHER_FN = ctypes.CFUNCTYPE(c_int, c_void_p, c_size_t, c_int, c_int, c_void_p, c_void_p)


class StreamConfig(Structure):
    _fields_ = [("block_size", c_int), ("enable_prefetch", c_int), ("reuse_resident", c_int),
                ("poison_on_release", c_int), ("n_slots", c_int), ("shard_world", c_int),
                ("shard_rank", c_int), ("gather", GATHER_FN), ("gather_user", c_void_p),
                ("shard_slab", c_int)]


class StreamStats(Structure):
    _fields_ = [("h2d_bytes", c_uint64), ("copies", c_uint64), ("reuses", c_uint64),
                ("acquires", c_uint64), ("releases", c_uint64), ("gathers", c_uint64)]


class KernelTime(Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", c_uint64), ("total_ms", ctypes.c_double),
                ("work", ctypes.c_double)]


class GemmPlanInfo(Structure):
    _fields_ = [("stream_k", ctypes.c_int32), ("pairs", ctypes.c_int32),
                ("units", ctypes.c_int32), ("split_tiles", ctypes.c_int32),
                ("total_steps", c_int64), ("max_pair_steps", c_int64),
                ("min_pair_steps", c_int64), ("covered", ctypes.c_int32),
                ("fixup_tiles", ctypes.c_int32)]


class HsNf4Error(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"[{status}] {detail}")
        self.status = status
        self.detail = detail


_lib = None

_SIGS = {
    "hsnf4_status_string": ([c_int], c_char_p),
    "hsnf4_last_error": ([c_char_p, c_size_t], c_int),
    "hsnf4_device_status": ([c_void_p, POINTER(c_uint32)], c_int),
    "hsnf4_inject_fault": ([c_char_p], c_int),
    "hsnf4_selftest_stall": ([c_void_p], c_int),
    "hsnf4_profile": ([c_int], c_int),
    "hsnf4_profile_kinds": ([c_uint32], c_int),
    "hsnf4_kernel_launches": ([], c_uint64),
    "hsnf4_profile_read": ([POINTER(KernelTime), c_int], c_int),
    "nf4_codebook": ([POINTER(c_float)], c_int),
    "nf4_quantize_pack": ([c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p], c_int),
    "nf4_dequant": ([c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p], c_int),
    "lora_merge": ([POINTER(Nf4WeightC), c_void_p, c_void_p, c_int, c_float, c_void_p, c_void_p],
                   c_int),
    "decoder_rmsnorm_fwd": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                             c_float, c_void_p], c_int),
    "decoder_rmsnorm_bwd": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_int64, c_int64, c_float, c_void_p], c_int),
    "decoder_swiglu_fwd": ([c_void_p, c_void_p, c_void_p, c_int64, c_void_p], c_int),
    "decoder_swiglu_bwd": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_void_p],
                           c_int),
    "decoder_add": ([c_void_p, c_void_p, c_void_p, c_int64, c_void_p], c_int),
    "decoder_attention_fwd": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int,
                               c_int, c_void_p], c_int),
    "decoder_attention_scratch_bytes": ([c_int64, c_int], c_size_t),
    "decoder_attention_bwd": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int, c_int,
                               c_void_p], c_int),
    "lora_dropout_apply": ([c_void_p, c_int64, c_int64, c_float, c_uint64, c_uint64, c_void_p,
                            c_void_p], c_int),
    "lora_linear_fwd_workspace": ([c_int64, c_int64, c_int64, c_int], c_size_t),
    "lora_linear_bwd_workspace": ([c_int64, c_int64, c_int64, c_int], c_size_t),
    "lora_linear_fwd": ([POINTER(Nf4WeightC), c_void_p, c_int64, c_void_p, c_void_p, c_int, c_float,
                         c_void_p, c_void_p, c_void_p, c_size_t, c_void_p], c_int),
    "lora_linear_bwd": ([POINTER(Nf4WeightC), c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_int,
                         c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                         c_void_p], c_int),
    "lora_linear_fwd_noalloc": ([POINTER(Nf4WeightC), c_void_p, c_int64, c_void_p, c_void_p, c_int,
                                 c_float, c_void_p, c_void_p, c_void_p], c_int),
    "hsnf4_gemm_plan": ([c_int, POINTER(c_int64), POINTER(c_int64), c_int, c_int64, c_int,
                         POINTER(GemmPlanInfo)], c_int),
    "lora_group_fwd_workspace": ([POINTER(FwdArgs), c_int, c_int64, c_int], c_size_t),
    "lora_group_bwd_workspace": ([POINTER(BwdArgs), c_int, c_int64, c_int], c_size_t),
    "lora_group_fwd": ([POINTER(FwdArgs), c_int, c_int64, c_int, c_float, c_void_p, c_size_t,
                        c_void_p], c_int),
    "lora_group_bwd": ([POINTER(BwdArgs), c_int, c_int64, c_int, c_float, c_void_p, c_size_t,
                        c_void_p], c_int),
    "stream_layer_bytes": ([POINTER(LayerDesc), POINTER(c_size_t)], c_int),
    "stream_layer_offsets": ([POINTER(LayerDesc), c_int, POINTER(c_size_t), POINTER(c_size_t)], c_int),
    "stream_slab_bytes": ([POINTER(LayerDesc), c_int, POINTER(c_size_t)], c_int),
    "stream_ring_bytes": ([POINTER(LayerDesc), c_int, c_int, POINTER(c_size_t)], c_int),
    "stream_slot_bytes": ([POINTER(LayerDesc), c_int, c_int, POINTER(c_size_t)], c_int),
    "stream_prefetch_ahead": ([c_void_p, POINTER(c_int), c_int, POINTER(c_int)], c_int),
    "stream_shard_range": ([c_size_t, c_int, c_int, POINTER(c_size_t), POINTER(c_size_t),
                            POINTER(c_size_t)], c_int),
    "stream_shard_slab_layout": ([POINTER(LayerDesc), c_int, c_int, c_int, c_int, c_int,
                                  POINTER(c_size_t), POINTER(c_size_t), POINTER(c_size_t)], c_int),
    "stream_slot_bytes_sharded": ([POINTER(LayerDesc), c_int, c_int, c_int, POINTER(c_size_t)],
                                  c_int),
    "stream_create": ([c_void_p, c_size_t, POINTER(LayerDesc), c_int, POINTER(StreamConfig), c_void_p,
                       c_size_t, c_void_p, POINTER(c_void_p)], c_int),
    "stream_num_blocks": ([c_void_p], c_int),
    "stream_block_prefetch": ([c_void_p, c_int], c_int),
    "stream_block_acquire": ([c_void_p, c_int, c_void_p, POINTER(Nf4WeightC), c_int], c_int),
    "stream_block_acquire_host": ([c_void_p, c_int, c_int], c_int),
    "stream_block_release": ([c_void_p, c_int, c_void_p], c_int),
    "stream_stats": ([c_void_p, POINTER(StreamStats)], c_int),
    "stream_destroy": ([c_void_p], c_int),
}

EXPORTS = tuple(_SIGS)


def lib():
    """Load libhsnf4.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m host_streamed_nf4_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def last_error() -> str:
    buf = ctypes.create_string_buffer(512)
    lib().hsnf4_last_error(buf, 512)
    return buf.value.decode(errors="replace")


def _check(rc: int):
    if rc != OK:
        raise HsNf4Error(rc, last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, device=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ------------------------------------------------------------------ diagnostics

def device_status(stream=None) -> int:
    flags = c_uint32(0)
    rc = lib().hsnf4_device_status(_stream(stream), ctypes.byref(flags))
    if rc not in (OK, ERR_DEVICE):
        _check(rc)
    return int(flags.value)


def kernel_launches() -> int:
    """Kernels this library has launched in this process so far."""
    return int(lib().hsnf4_kernel_launches())


PROFILE_KINDS = ("lora_gemm_fwd", "lora_gemm_dx", "nf4_dequant", "lora_merge", "lora_project",
                 "lora_grad")


def profile(enable: bool, kinds=None):
    """Start (clearing) or stop kernel timing; `kinds`, a subset of
    PROFILE_KINDS, times only those launches."""
    if enable and kinds is not None:
        mask = 0
        for k in kinds:
            mask |= 1 << PROFILE_KINDS.index(k)
        _check(lib().hsnf4_profile_kinds(mask))
    else:
        _check(lib().hsnf4_profile(int(bool(enable))))


def gemm_plan(mode: str, shapes, T: int, r: int) -> dict:
    """The fused GEMM's work plan for a group of (n_out, k_in) shapes (host
    only): mode "fwd" or "dx"."""
    n = len(shapes)
    n_out = (c_int64 * n)(*[s[0] for s in shapes])
    k_in = (c_int64 * n)(*[s[1] for s in shapes])
    info = GemmPlanInfo()
    _check(lib().hsnf4_gemm_plan({"fwd": 0, "dx": 1}[mode], n_out, k_in, n, T, r,
                                 ctypes.byref(info)))
    return {f[0]: getattr(info, f[0]) for f in GemmPlanInfo._fields_}


def profile_read() -> dict:
    """{kernel name: {"launches", "total_ms", "work"}} since profile(True)."""
    out = (KernelTime * 8)()
    n = lib().hsnf4_profile_read(out, 8)
    if n < 0:
        _check(-n)
    return {out[i].name.decode(): {"launches": int(out[i].launches), "total_ms": out[i].total_ms,
                                   "work": out[i].work} for i in range(n)}


def selftest_stall(stream=None):
    _check(lib().hsnf4_selftest_stall(_stream(stream)))


def inject_fault(site: str | None):
    _check(lib().hsnf4_inject_fault(site.encode() if site else None))


def codebook() -> list[float]:
    out = (c_float * 16)()
    _check(lib().nf4_codebook(out))
    return list(out)


# ------------------------------------------------------------------ NF4

@dataclass
class Nf4Weight:
    """An NF4 weight in device memory (codes uint8, absmax fp32)."""
    codes: torch.Tensor
    absmax: torch.Tensor
    n_out: int
    k_in: int

    def c(self) -> Nf4WeightC:
        return Nf4WeightC(self.codes.data_ptr(), self.absmax.data_ptr(), self.n_out, self.k_in,
                          BASE_NF4, 0)


@dataclass
class Bf16Weight:
    """A dense bf16 base weight [n_out, k_in] in device memory (the
    quantization="bf16_bitwise" base: streamed, never dequantized)."""
    w: torch.Tensor

    @property
    def n_out(self) -> int:
        return self.w.shape[0]

    @property
    def k_in(self) -> int:
        return self.w.shape[1]

    def c(self) -> Nf4WeightC:
        _need(self.w, "w", torch.bfloat16)
        return Nf4WeightC(self.w.data_ptr(), None, self.n_out, self.k_in, BASE_BF16, 0)


def nf4_quantize_pack(w: torch.Tensor, codes=None, absmax=None, stream=None) -> Nf4Weight:
    _need(w, "w", torch.bfloat16)
    n, k = w.shape
    if codes is None:
        codes = torch.empty(n * k // 2, dtype=torch.uint8, device=w.device)
    if absmax is None:
        absmax = torch.empty(n * k // 64, dtype=torch.float32, device=w.device)
    _check(lib().nf4_quantize_pack(_ptr(w), n, k, _ptr(codes), _ptr(absmax), _stream(stream)))
    return Nf4Weight(codes, absmax, n, k)


def nf4_dequant(W: Nf4Weight, out=None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(W.n_out, W.k_in, dtype=torch.bfloat16, device=W.codes.device)
    _check(lib().nf4_dequant(_ptr(W.codes), _ptr(W.absmax), W.n_out, W.k_in, _ptr(out),
                             _stream(stream)))
    return out


def lora_merge(W, A: torch.Tensor, B: torch.Tensor, alpha: float, out=None, stream=None):
    """W' = deq(W) + (alpha/r) B A as a bf16 [n_out, k_in] tensor (merge_and_unload)."""
    r = A.shape[0]
    dev = A.device
    if out is None:
        out = torch.empty(W.n_out, W.k_in, dtype=torch.bfloat16, device=dev)
    _check(lib().lora_merge(_weight_arg(W), _ptr(A), _ptr(B), r, float(alpha), _ptr(out),
                            _stream(stream)))
    return out


# ------------------------------------------------------------------ decoder glue

def _pp(t):
    return None if t is None else _ptr(t)


def rmsnorm_fwd(x, g, eps, res=None, h_out=None, y=None, stream=None):
    """y = rmsnorm(x [+ res]) (bf16 [T, n]); with res, h_out receives x + res."""
    T, n = x.shape
    if y is None:
        y = torch.empty_like(x)
    if res is not None and h_out is None:
        h_out = torch.empty_like(x)
    _check(lib().decoder_rmsnorm_fwd(_ptr(x), _pp(res), _ptr(g), _pp(h_out), _ptr(y), T, n,
                                     float(eps), _stream(stream)))
    return (y, h_out) if res is not None else y


def rmsnorm_bwd(x, g, dys, eps, dres=None, dx=None, stream=None):
    """dx = dres + drmsnorm(x)/dx . sum(dys) (1..3 bf16 branch gradients)."""
    T, n = x.shape
    if dx is None:
        dx = torch.empty_like(x)
    d = list(dys) + [None] * (3 - len(dys))
    _check(lib().decoder_rmsnorm_bwd(_ptr(x), _ptr(g), _ptr(d[0]), _pp(d[1]), _pp(d[2]), _pp(dres),
                                     _ptr(dx), T, n, float(eps), _stream(stream)))
    return dx


def swiglu_fwd(a, b, m=None, stream=None):
    if m is None:
        m = torch.empty_like(a)
    _check(lib().decoder_swiglu_fwd(_ptr(a), _ptr(b), _ptr(m), a.numel(), _stream(stream)))
    return m


def swiglu_bwd(a, b, dm, da=None, db=None, stream=None):
    da = torch.empty_like(a) if da is None else da
    db = torch.empty_like(a) if db is None else db
    _check(lib().decoder_swiglu_bwd(_ptr(a), _ptr(b), _ptr(dm), _ptr(da), _ptr(db), a.numel(),
                                    _stream(stream)))
    return da, db


def add(x, y, out=None, stream=None):
    out = torch.empty_like(x) if out is None else out
    _check(lib().decoder_add(_ptr(x), _ptr(y), _ptr(out), x.numel(), _stream(stream)))
    return out


def attention_fwd(q, k, v, H, KV, o=None, lse=None, stream=None):
    T = q.shape[0]
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty(H, T, dtype=torch.float32, device=q.device) if lse is None else lse
    _check(lib().decoder_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), T, H, KV,
                                       _stream(stream)))
    return o, lse


def attention_scratch_bytes(T: int, H: int) -> int:
    return int(lib().decoder_attention_scratch_bytes(T, H))


def attention_bwd(q, k, v, o, lse, dout, H, KV, dq=None, dk=None, dv=None, scratch=None,
                  stream=None):
    T = q.shape[0]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if scratch is None:
        scratch = torch.empty(attention_scratch_bytes(T, H), dtype=torch.uint8, device=q.device)
    _check(lib().decoder_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                       _ptr(dq), _ptr(dk), _ptr(dv), _ptr(scratch), T, H, KV,
                                       _stream(stream)))
    return dq, dk, dv


# ------------------------------------------------------------------ LoRA linear

def fwd_workspace_bytes(T, n_out, k_in, r) -> int:
    return int(lib().lora_linear_fwd_workspace(T, n_out, k_in, r))


def bwd_workspace_bytes(T, n_out, k_in, r) -> int:
    return int(lib().lora_linear_bwd_workspace(T, n_out, k_in, r))


def _weight_arg(W):
    return ctypes.byref(_wc(W))


def lora_linear_fwd(W, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                    Y=None, t_save=None, workspace=None, stream=None):
    """Y = X deq(W)^T + (alpha/r) (X A^T) B^T.  Returns (Y bf16 [T, n_out], t fp32 [T, r])."""
    n_out, k_in = W.n_out, W.k_in
    T, r = X.shape[0], A.shape[0]
    if Y is None:
        Y = torch.empty(T, n_out, dtype=torch.bfloat16, device=X.device)
    if t_save is None:
        t_save = torch.empty(T, r, dtype=torch.float32, device=X.device)
    ws = fwd_workspace_bytes(T, n_out, k_in, r)
    if workspace is None:
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=X.device)
    _check(lib().lora_linear_fwd(_weight_arg(W), _ptr(X), T, _ptr(A), _ptr(B), r, float(alpha),
                                 _ptr(Y), _ptr(t_save), _ptr(workspace), workspace.numel(),
                                 _stream(stream)))
    return Y, t_save


def lora_linear_fwd_noalloc(W, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                            Y=None, t_save=None, stream=None):
    """The forward without a workspace argument, for callers that cannot
    allocate device memory: the library's built-in 64 MiB scratch is used.
    (The output buffers passed here may be preallocated by the caller.)"""
    n_out = W.n_out
    T, r = X.shape[0], A.shape[0]
    if Y is None:
        Y = torch.empty(T, n_out, dtype=torch.bfloat16, device=X.device)
    if t_save is None:
        t_save = torch.empty(T, r, dtype=torch.float32, device=X.device)
    _check(lib().lora_linear_fwd_noalloc(_weight_arg(W), _ptr(X), T, _ptr(A), _ptr(B), r,
                                         float(alpha), _ptr(Y), _ptr(t_save), _stream(stream)))
    return Y, t_save


def lora_linear_bwd(W, X, t_save, A, B, dY, alpha: float, dX=None, dA=None, dB=None,
                    workspace=None, stream=None):
    """Returns (dX bf16 [T, k_in], dA fp32 [r, k_in], dB fp32 [n_out, r])."""
    n_out, k_in = W.n_out, W.k_in
    T, r = X.shape[0], A.shape[0]
    dev = X.device
    if dX is None:
        dX = torch.empty(T, k_in, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(r, k_in, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(n_out, r, dtype=torch.float32, device=dev)
    ws = bwd_workspace_bytes(T, n_out, k_in, r)
    if workspace is None:
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    _check(lib().lora_linear_bwd(_weight_arg(W), _ptr(X), _ptr(t_save), T, _ptr(A), _ptr(B), r,
                                 float(alpha), _ptr(dY), _ptr(dX), _ptr(dA), _ptr(dB),
                                 _ptr(workspace), workspace.numel(), _stream(stream)))
    return dX, dA, dB


def _wc(W):
    return W.c() if isinstance(W, (Nf4Weight, Bf16Weight)) else W


def _p(t):
    return None if t is None else t.data_ptr()


def fwd_args(W, X, A, B, Y, t_save=None, dropout=None) -> FwdArgs:
    """One problem of a grouped forward (tensors are kept alive by the caller).
    dropout: (p, seed, offset) for the adapter branch, or None."""
    p, seed, off = dropout or (0.0, 0, 0)
    return FwdArgs(_wc(W), _p(X), _p(A), _p(B), _p(Y), _p(t_save), p, 0, seed, off)


def bwd_args(W, X, t_save, A, B, dY, dX, dA, dB, dropout=None) -> BwdArgs:
    p, seed, off = dropout or (0.0, 0, 0)
    return BwdArgs(_wc(W), _p(X), _p(t_save), _p(A), _p(B), _p(dY), _p(dX), _p(dA), _p(dB),
                   p, 0, seed, off)


def lora_dropout_apply(X: torch.Tensor, p: float, seed: int, offset: int, out=None,
                       stream=None) -> torch.Tensor:
    """X_d = dropout(X) on the adapter branch's definition (bf16 [T, K])."""
    _need(X, "X", torch.bfloat16)
    T, K = X.shape
    if out is None:
        out = torch.empty_like(X)
    _check(lib().lora_dropout_apply(_ptr(X), T, K, float(p), seed, offset, _ptr(out),
                                    _stream(stream)))
    return out


def group_fwd_workspace_bytes(args, T, r) -> int:
    arr = (FwdArgs * len(args))(*args)
    return int(lib().lora_group_fwd_workspace(arr, len(args), T, r))


def group_bwd_workspace_bytes(args, T, r) -> int:
    arr = (BwdArgs * len(args))(*args)
    return int(lib().lora_group_bwd_workspace(arr, len(args), T, r))


def lora_group_fwd(args, T: int, r: int, alpha: float, workspace: torch.Tensor, stream=None):
    """Forward of len(args) independent LoRA linears in one grouped call."""
    arr = (FwdArgs * len(args))(*args)
    _check(lib().lora_group_fwd(arr, len(args), T, r, float(alpha), _ptr(workspace),
                                workspace.numel(), _stream(stream)))


def lora_group_bwd(args, T: int, r: int, alpha: float, workspace: torch.Tensor, stream=None):
    arr = (BwdArgs * len(args))(*args)
    _check(lib().lora_group_bwd(arr, len(args), T, r, float(alpha), _ptr(workspace),
                                workspace.numel(), _stream(stream)))


# ------------------------------------------------------------------ streamer

def layer_desc(shapes, base_format: int = 0) -> LayerDesc:
    """shapes: [(n_out, k_in), ...] of one layer's projections; base_format
    BASE_NF4 (codes + absmax) or BASE_BF16 (dense bf16 weights)."""
    d = LayerDesc()
    d.n_proj = len(shapes)
    d.base_format = base_format
    for i, (n, k) in enumerate(shapes):
        d.n_out[i] = n
        d.k_in[i] = k
    return d


def layer_bytes(desc: LayerDesc) -> int:
    out = c_size_t(0)
    _check(lib().stream_layer_bytes(ctypes.byref(desc), ctypes.byref(out)))
    return out.value


def layer_offsets(desc: LayerDesc, proj: int):
    co, ao = c_size_t(0), c_size_t(0)
    _check(lib().stream_layer_offsets(ctypes.byref(desc), proj, ctypes.byref(co), ctypes.byref(ao)))
    return co.value, ao.value


def _desc_array(descs):
    arr = (LayerDesc * len(descs))(*descs)
    return arr


def slab_bytes(descs) -> int:
    out = c_size_t(0)
    _check(lib().stream_slab_bytes(_desc_array(descs), len(descs), ctypes.byref(out)))
    return out.value


def ring_bytes(descs, block_size: int, n_slots: int = 2, shard_world: int = 0) -> int:
    """Device bytes of an n_slots ring; shard_world >= 1: of a sharded stream."""
    out = c_size_t(0)
    if shard_world >= 1:
        _check(lib().stream_slot_bytes_sharded(_desc_array(descs), len(descs), block_size,
                                               shard_world, ctypes.byref(out)))
    else:
        _check(lib().stream_slot_bytes(_desc_array(descs), len(descs), block_size,
                                       ctypes.byref(out)))
    return out.value * n_slots


def shard_range(block_bytes: int, world: int, rank: int):
    """(stride S, offset, length) of rank's shard of a block shared by world ranks."""
    S, off, n = c_size_t(0), c_size_t(0), c_size_t(0)
    _check(lib().stream_shard_range(block_bytes, world, rank, ctypes.byref(S), ctypes.byref(off),
                                    ctypes.byref(n)))
    return S.value, off.value, n.value


def shard_slab_layout(descs, block_size: int, world: int, rank: int):
    """Rank's shard slab: ([(offset in the shard slab, length) per block], total bytes)."""
    arr = _desc_array(descs)
    total = c_size_t(0)
    _check(lib().stream_shard_slab_layout(arr, len(descs), block_size, world, rank, -1, None,
                                          None, ctypes.byref(total)))
    n_blocks = (len(descs) + block_size - 1) // block_size
    out = []
    for b in range(n_blocks):
        off, n = c_size_t(0), c_size_t(0)
        _check(lib().stream_shard_slab_layout(arr, len(descs), block_size, world, rank, b,
                                              ctypes.byref(off), ctypes.byref(n), None))
        out.append((off.value, n.value))
    return out, total.value


class Streamer:
    """Pinned-host NF4 stack -> 2-slot VRAM ring, prefetched one block ahead.

    shard=(rank, world, gather): stream 1/world of every block over this
    rank's link; gather(slot_offset, shard_bytes, world, block) must enqueue,
    on the current CUDA stream (the copy stream), the in-place all-gather of
    the ring bytes [slot_offset, slot_offset + world * shard_bytes).
    shard_slab: the slab holds only this rank's shards (shard_slab_layout)."""

    def __init__(self, slab: torch.Tensor, descs, block_size: int, ring: torch.Tensor,
                 copy_stream: torch.cuda.Stream, enable_prefetch=True, reuse_resident=True,
                 poison_on_release=False, n_slots=2, shard=None, shard_slab=False):
        _need(slab, "slab", torch.uint8, device=False)
        if not slab.is_pinned():
            raise ValueError("slab must be page-locked (pin_memory)")
        _need(ring, "ring", torch.uint8)
        self.descs = list(descs)
        self._arr = _desc_array(self.descs)
        cfg = StreamConfig(block_size, int(bool(enable_prefetch)), int(bool(reuse_resident)),
                           int(bool(poison_on_release)), int(n_slots))
        self._gather_error = None
        self._gather_cb = None
        if shard is not None:
            rank, world, fn = shard
            base = ring.data_ptr()

            def _cb(slot, shard_bytes, world_, block, stream, user):
                try:
                    with torch.cuda.stream(copy_stream):
                        fn(slot - base, shard_bytes, world_, block)
                    return 0
                except Exception as e:  # reported through the library's status
                    self._gather_error = e
                    return 1

            self._gather_cb = GATHER_FN(_cb)
            cfg.shard_world, cfg.shard_rank = world, rank
            cfg.gather = self._gather_cb
            cfg.shard_slab = int(bool(shard_slab))
        self.n_slots = n_slots
        h = c_void_p()
        _check(lib().stream_create(_ptr(slab), slab.numel(), self._arr, len(self.descs),
                                   ctypes.byref(cfg), _ptr(ring), ring.numel(),
                                   ctypes.c_void_p(copy_stream.cuda_stream), ctypes.byref(h)))
        self._h = h
        self.slab, self.ring, self.copy_stream = slab, ring, copy_stream
        self.block_size = block_size
        self.n_blocks = lib().stream_num_blocks(h)

    def _check(self, rc: int):
        err, self._gather_error = self._gather_error, None
        if rc != 0 and err is not None:
            raise HsNf4Error(rc, f"{last_error()} ({type(err).__name__}: {err})") from err
        _check(rc)

    def prefetch(self, b: int):
        self._check(lib().stream_block_prefetch(self._h, b))

    def prefetch_ahead(self, upcoming) -> int:
        arr = (c_int * len(upcoming))(*upcoming)
        issued = c_int(0)
        self._check(lib().stream_prefetch_ahead(self._h, arr, len(upcoming), ctypes.byref(issued)))
        return issued.value

    def acquire(self, b: int, stream=None):
        first = b * self.block_size
        n = sum(d.n_proj for d in self.descs[first:first + self.block_size])
        out = (Nf4WeightC * n)()
        self._check(lib().stream_block_acquire(self._h, b, _stream(stream), out, n))
        return list(out)

    def acquire_host(self, b: int, timeout_ms: int):
        _check(lib().stream_block_acquire_host(self._h, b, timeout_ms))

    def release(self, b: int, stream=None):
        _check(lib().stream_block_release(self._h, b, _stream(stream)))

    def stats(self) -> dict:
        s = StreamStats()
        _check(lib().stream_stats(self._h, ctypes.byref(s)))
        return {f: int(getattr(s, f)) for f, _ in StreamStats._fields_}

    def close(self):
        if self._h:
            rc = lib().stream_destroy(self._h)
            self._h = None
            _check(rc)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
