"""ctypes binding of librf (include/rf.h): argument marshalling only.

Every step of the path runs in librf's CUDA kernels; this module only turns
torch tensors into device pointers and the current stream into a
cudaStream_t.  Importing it fails loudly when librf.so has not been built.

Pages the method is described on: the "RainFusion Attention" user guide
(vllm-omni docs), the xllm pull request "feat: add RainFusion sparse
attention for wan2.2" (#1867), the CANN "aclnnRainFusionAttention" API page
and the RainFusion2.0 abstract.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Iterable, List, Optional, Sequence, Tuple

import torch

# RF_LIBRARY may name another build of librf (same ABI), e.g. to compare builds.
LIB_PATH = os.environ.get("RF_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "librf.so")

RF_OK = 0
STATUS_NAMES = {0: "RF_OK", 1: "RF_ERR_INVALID_ARG", 2: "RF_ERR_UNSUPPORTED_DEVICE",
                3: "RF_ERR_WORKSPACE_TOO_SMALL", 4: "RF_ERR_CUDA", 5: "RF_ERR_DEVICE_FAULT",
                6: "RF_ERR_UNSUPPORTED"}
LAYOUTS = {"BNSD": 0, "TND": 1}
DTYPES = {"bf16": 0, "fp16": 1}
ORDERS = {"tile": 0, "frame_pair": 1}   # rf_token_order_t
PRECISIONS = {"native": 0, "mix": 1, "fp8": 2, "mxfp4": 3}   # rf_precision_t
TORCH_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}
POOL_MODES = {"from_ws": 0, "recompute": 1}

EXPORTED = ("rf_plan_create", "rf_plan_info", "rf_plan_seq_info", "rf_rearrange", "rf_pool_select",
            "rf_block_sparse_attn", "rf_inverse_rearrange", "rf_forward", "rf_check_device_status",
            "rf_plan_destroy", "rf_status_string", "rf_last_error", "rf_plan_permutation",
            "rf_selftest_exp2", "rf_pool_select_noalloc", "rf_plan_create_ex", "rf_quantize_qk",
            "rf_selftest_expired_wait", "rf_quantize_mx", "rf_quantize")


class RfError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")
        self.status = status


class SeqGeom(ctypes.Structure):
    _fields_ = [("prefix_len", ctypes.c_int32), ("t", ctypes.c_int32), ("h", ctypes.c_int32),
                ("w", ctypes.c_int32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("rows_total", ctypes.c_int64), ("t_qblk", ctypes.c_int64),
                ("max_kv_blocks", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64),
                ("pooled_blocks", ctypes.c_int64), ("kept_flops_upper", ctypes.c_int64),
                ("ws_pooled_q", ctypes.c_int64), ("ws_pooled_k", ctypes.c_int64),
                ("n_seqs", ctypes.c_int32), ("n1", ctypes.c_int32), ("n2", ctypes.c_int32),
                ("d", ctypes.c_int32), ("precision", ctypes.c_int32), ("token_order", ctypes.c_int32),
                ("ws_q8", ctypes.c_int64), ("ws_k8", ctypes.c_int64),
                ("ws_q_scale", ctypes.c_int64), ("ws_k_scale", ctypes.c_int64),
                ("ws_q_mx", ctypes.c_int64), ("ws_k_mx", ctypes.c_int64), ("ws_v_mx", ctypes.c_int64),
                ("ws_v8", ctypes.c_int64), ("ws_v_exp", ctypes.c_int64),
                ("pooled_k_blocks", ctypes.c_int64)]


class PlanOptions(ctypes.Structure):
    _fields_ = [("token_order", ctypes.c_int32), ("precision", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 6)]


class SeqInfo(ctypes.Structure):
    _fields_ = [("row_offset", ctypes.c_int64), ("length", ctypes.c_int64), ("lp", ctypes.c_int64),
                ("sparse", ctypes.c_int64), ("promoted", ctypes.c_int64), ("n_pb", ctypes.c_int32),
                ("nb", ctypes.c_int32), ("ns", ctypes.c_int32), ("k", ctypes.c_int32),
                ("qblk_offset", ctypes.c_int32), ("dense", ctypes.c_int32),
                ("n_pb_kv", ctypes.c_int32), ("nb_kv", ctypes.c_int32), ("ns_kv", ctypes.c_int32),
                ("k_kv", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m block_sparse_video_rearrange_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "rf_plan_create": [ctypes.POINTER(SeqGeom), i32, i32, i32, i32, i32, i32, i32, ctypes.c_double,
                           i32, i32, ctypes.POINTER(vp)],
        "rf_plan_create_ex": [ctypes.POINTER(SeqGeom), i32, i32, i32, i32, i32, i32, i32, ctypes.c_double,
                              i32, i32, ctypes.POINTER(PlanOptions), ctypes.POINTER(vp)],
        "rf_quantize_qk": [vp, vp, vp, vp, sz, vp],
        "rf_quantize_mx": [vp, vp, vp, vp, vp, sz, vp],
        "rf_quantize": [vp, vp, vp, vp, vp, sz, vp],
        "rf_selftest_expired_wait": [vp, vp, sz, vp],
        "rf_plan_info": [vp, ctypes.POINTER(PlanInfo)],
        "rf_plan_seq_info": [vp, i32, ctypes.POINTER(SeqInfo)],
        "rf_rearrange": [vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "rf_pool_select": [vp, vp, vp, vp, vp, vp, sz, i32, vp],
        "rf_block_sparse_attn": [vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, vp, vp, sz, vp],
        "rf_inverse_rearrange": [vp, vp, vp, vp],
        "rf_forward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, sz, vp],
        "rf_check_device_status": [vp, vp, ctypes.POINTER(ctypes.c_uint32), vp],
        "rf_plan_destroy": [vp],
        "rf_selftest_exp2": [vp, vp, vp, ctypes.c_int64, vp],
        "rf_pool_select_noalloc": [vp, vp, vp, vp, vp, vp],
        "rf_plan_permutation": [vp, i32, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64],
        "rf_status_string": [i32],
        "rf_last_error": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int32
    lib.rf_plan_destroy.restype = None
    lib.rf_status_string.restype = ctypes.c_char_p
    lib.rf_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _check(status: int, where: str) -> None:
    if status != RF_OK:
        raise RfError(status, where, _lib.rf_last_error().decode())


class Plan:
    """Host-side plan: validated geometry and sizes (no device memory)."""

    def __init__(self, seqs: Sequence[Tuple[int, int, int, int]], n1: int, n2: int, d: int,
                 layout: str = "BNSD", dtype: str = "bf16", sparsity: float = 0.8, batch: int = 1,
                 block_q: int = 128, block_kv: int = 128, order: str = "tile", precision: str = "native"):
        arr = (SeqGeom * max(1, len(seqs)))(*[SeqGeom(*map(int, s)) for s in seqs])
        handle = ctypes.c_void_p()
        if order not in ORDERS:
            raise ValueError(f"order must be one of {sorted(ORDERS)}")
        if precision not in PRECISIONS:
            raise ValueError(f"precision must be one of {sorted(PRECISIONS)}")
        opts = PlanOptions(ORDERS[order], PRECISIONS[precision])
        _check(_lib.rf_plan_create_ex(arr, len(seqs), batch, n1, n2, d, LAYOUTS[layout], DTYPES[dtype],
                                      float(sparsity), block_q, block_kv, ctypes.byref(opts),
                                      ctypes.byref(handle)),
               "rf_plan_create_ex")
        self.order = order
        self.precision = precision
        self.block_q, self.block_kv = int(block_q), int(block_kv)
        self._h = handle
        self._lib = _lib  # kept so that destruction at interpreter exit still finds it
        self.layout, self.dtype, self.sparsity, self.batch = layout, dtype, float(sparsity), batch
        self.seqs = [tuple(map(int, s)) for s in seqs]
        info = PlanInfo()
        _check(_lib.rf_plan_info(self._h, ctypes.byref(info)), "rf_plan_info")
        self.info = info
        self.seq_info: List[SeqInfo] = []
        for i in range(len(seqs)):
            si = SeqInfo()
            _check(_lib.rf_plan_seq_info(self._h, i, ctypes.byref(si)), "rf_plan_seq_info")
            self.seq_info.append(si)

    def __del__(self):
        h, lib_ = getattr(self, "_h", None), getattr(self, "_lib", None)
        if h is not None and h.value and lib_ is not None:
            lib_.rf_plan_destroy(h)
            self._h = None

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    @property
    def n1(self) -> int:
        return self.info.n1

    @property
    def n2(self) -> int:
        return self.info.n2

    @property
    def d(self) -> int:
        return self.info.d

    @property
    def torch_dtype(self) -> torch.dtype:
        return TORCH_DTYPES[self.dtype]

    def tensor_shape(self, heads: int) -> Tuple[int, ...]:
        if self.layout == "BNSD":
            return (self.batch, heads, int(self.seq_info[0].length), self.d)
        return (int(self.info.rows_total), heads, self.d)

    def select_shapes(self) -> Tuple[Tuple[int, int, int], Tuple[int, int]]:
        t, n, m = int(self.info.t_qblk), self.n1, int(self.info.max_kv_blocks)
        return (t, n, m), (t, n)

    @property
    def workspace_bytes(self) -> int:
        return int(self.info.workspace_bytes)

    def permutation(self, seq: int = 0):
        """src[r] = original row of rearranged row r of sequence `seq` (host-side arithmetic)."""
        import numpy as np
        n = int(self.seq_info[seq].length)
        out = np.empty(n, dtype=np.int64)
        _check(_lib.rf_plan_permutation(self._h, seq, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n),
               "rf_plan_permutation")
        return out

    def seq_info_all(self) -> List[SeqInfo]:
        """Geometry of every sequence instance in q-block order (BNSD: one per batch element)."""
        if self.layout == "TND":
            return list(self.seq_info)
        out = []
        base = self.seq_info[0]
        nblk = base.n_pb + base.nb
        for bi in range(self.batch):
            si = SeqInfo()
            ctypes.pointer(si)[0] = base
            si.qblk_offset = bi * nblk
            out.append(si)
        return out


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("librf takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _expect(t: torch.Tensor, shape, dtype, name: str) -> None:
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name}: expected {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")


def rearrange(plan: Plan, q, k, v, q_r, k_r, v_r, ws, stream=None) -> None:
    """Permute Q, K, V (one launch) and write the block means of Q and K into ws."""
    for t, h, nm in ((q, plan.n1, "q"), (k, plan.n2, "k"), (v, plan.n2, "v"), (q_r, plan.n1, "q_r"),
                     (k_r, plan.n2, "k_r"), (v_r, plan.n2, "v_r")):
        _expect(t, plan.tensor_shape(h), plan.torch_dtype, nm)
    _check(_lib.rf_rearrange(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(q_r), _ptr(k_r), _ptr(v_r),
                             _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "rf_rearrange")


def pool_select(plan: Plan, q_r, k_r, select_idx, select_num, ws, pool_mode: str = "from_ws",
                stream=None) -> None:
    """Rank key blocks per query block; write selectIdx / selectNum."""
    si, sn = plan.select_shapes()
    _expect(select_idx, si, torch.int32, "select_idx")
    _expect(select_num, sn, torch.int32, "select_num")
    _check(_lib.rf_pool_select(plan.handle, _ptr(q_r), _ptr(k_r), _ptr(select_idx), _ptr(select_num),
                               _ptr(ws), ws.numel() * ws.element_size(), POOL_MODES[pool_mode],
                               _stream(stream)), "rf_pool_select")


def pool_select_noalloc(plan: Plan, q_r, k_r, select_idx, select_num, stream=None) -> None:
    """Selection without any device allocation: the scratch is a static array
    inside librf (32 MiB per device, set up by the first call on a device).
    For callers that cannot allocate device memory; same result as
    pool_select(..., pool_mode="recompute").  Concurrent calls on one device race."""
    si, sn = plan.select_shapes()
    _expect(select_idx, si, torch.int32, "select_idx")
    _expect(select_num, sn, torch.int32, "select_num")
    _check(_lib.rf_pool_select_noalloc(plan.handle, _ptr(q_r), _ptr(k_r), _ptr(select_idx), _ptr(select_num),
                                       _stream(stream)), "rf_pool_select_noalloc")


def block_sparse_attn(plan: Plan, q_r, k_r, v_r, select_idx, select_num, scale: float, o_r, ws,
                      inner_precise: int = 0, stream=None) -> None:
    """Softmax(scale Q K^T) V over the selected blocks (rearranged order)."""
    _expect(o_r, plan.tensor_shape(plan.n1), plan.torch_dtype, "o_r")
    _check(_lib.rf_block_sparse_attn(plan.handle, _ptr(q_r), _ptr(k_r), _ptr(v_r), _ptr(select_idx),
                                     _ptr(select_num), float(scale), int(inner_precise), _ptr(o_r),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "rf_block_sparse_attn")


def quantize_qk(plan: Plan, q_r, k_r, ws, stream=None) -> None:
    """Precision "mix": E4M3 copies of rearranged q_r / k_r and their scales into ws."""
    _expect(q_r, plan.tensor_shape(plan.n1), plan.torch_dtype, "q_r")
    _expect(k_r, plan.tensor_shape(plan.n2), plan.torch_dtype, "k_r")
    _check(_lib.rf_quantize_qk(plan.handle, _ptr(q_r), _ptr(k_r), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream(stream)), "rf_quantize_qk")


def quantize_mx(plan: Plan, q_r, k_r, v_r, ws, stream=None) -> None:
    """Precision "mxfp4": MXFP4-rounded copies of rearranged q_r / k_r / v_r into ws."""
    _expect(q_r, plan.tensor_shape(plan.n1), plan.torch_dtype, "q_r")
    _expect(k_r, plan.tensor_shape(plan.n2), plan.torch_dtype, "k_r")
    _expect(v_r, plan.tensor_shape(plan.n2), plan.torch_dtype, "v_r")
    _check(_lib.rf_quantize_mx(plan.handle, _ptr(q_r), _ptr(k_r), _ptr(v_r), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "rf_quantize_mx")


def quantize(plan: Plan, q_r, k_r, v_r, ws, stream=None) -> None:
    """Every quantized copy the plan's precision needs ("mix", "fp8", "mxfp4"), from
    rearranged q_r / k_r / v_r, into ws (v_r may be None for "mix")."""
    _expect(q_r, plan.tensor_shape(plan.n1), plan.torch_dtype, "q_r")
    _expect(k_r, plan.tensor_shape(plan.n2), plan.torch_dtype, "k_r")
    if v_r is not None:
        _expect(v_r, plan.tensor_shape(plan.n2), plan.torch_dtype, "v_r")
    _check(_lib.rf_quantize(plan.handle, _ptr(q_r), _ptr(k_r), _ptr(v_r), _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "rf_quantize")


def inverse_rearrange(plan: Plan, o_r, o, stream=None) -> None:
    """Scatter the output back to the original token order."""
    _expect(o, plan.tensor_shape(plan.n1), plan.torch_dtype, "o")
    _check(_lib.rf_inverse_rearrange(plan.handle, _ptr(o_r), _ptr(o), _stream(stream)),
           "rf_inverse_rearrange")


def selftest_exp2(x: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(polynomial 2^x, ex2.approx 2^x) of a float32 device tensor, from the kernel's own code paths."""
    assert x.dtype == torch.float32 and x.is_cuda
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _check(_lib.rf_selftest_exp2(_ptr(x), _ptr(yp), _ptr(ym), x.numel(), _stream(stream)), "rf_selftest_exp2")
    return yp, ym


def selftest_expired_wait(plan: Plan, ws, stream=None) -> None:
    """Provoke one expired bounded wait (about 1 s on the device) recorded in ws's status words."""
    _check(_lib.rf_selftest_expired_wait(plan.handle, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "rf_selftest_expired_wait")


def check_device_status(plan: Plan, ws, stream=None) -> Tuple[int, Tuple[int, int]]:
    """Synchronise, read and clear the kernels' status words: (status, (bad_index, timeouts))."""
    flags = (ctypes.c_uint32 * 2)()
    st = _lib.rf_check_device_status(plan.handle, _ptr(ws), flags, _stream(stream))
    return st, (int(flags[0]), int(flags[1]))


def raise_on_device_fault(plan: Plan, ws, where: str, stream=None) -> None:
    """Synchronise, read and clear the status words in ws; raise RfError(RF_ERR_DEVICE_FAULT)
    if a kernel recorded an out-of-range selectIdx entry or an expired bounded wait."""
    st, flags = check_device_status(plan, ws, stream)
    if st != RF_OK:
        raise RfError(st, where, f"device status words: {flags[0]} bad selectIdx entries, "
                                 f"expired-wait bits {flags[1]:#x}")


class Buffers:
    """Device intermediates and outputs of one path invocation (owned by torch)."""

    def __init__(self, plan: Plan, device="cuda"):
        shp_q, shp_kv = plan.tensor_shape(plan.n1), plan.tensor_shape(plan.n2)
        dt = plan.torch_dtype
        self.q_r = torch.empty(shp_q, dtype=dt, device=device)
        self.k_r = torch.empty(shp_kv, dtype=dt, device=device)
        self.v_r = torch.empty(shp_kv, dtype=dt, device=device)
        self.o_r = torch.empty(shp_q, dtype=dt, device=device)
        self.o = torch.empty(shp_q, dtype=dt, device=device)
        si, sn = plan.select_shapes()
        self.select_idx = torch.empty(si, dtype=torch.int32, device=device)
        self.select_num = torch.empty(sn, dtype=torch.int32, device=device)
        self.ws = torch.zeros(max(256, plan.workspace_bytes) // 4 + 64, dtype=torch.int32, device=device)


def forward(plan: Plan, q, k, v, bufs: Buffers, scale: Optional[float] = None, stream=None) -> torch.Tensor:
    """The whole path in one librf call; returns bufs.o (original token order)."""
    if scale is None:
        scale = 1.0 / math.sqrt(plan.d)
    for t, h, nm in ((q, plan.n1, "q"), (k, plan.n2, "k"), (v, plan.n2, "v")):
        _expect(t, plan.tensor_shape(h), plan.torch_dtype, nm)
    b = bufs
    _check(_lib.rf_forward(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(b.q_r), _ptr(b.k_r), _ptr(b.v_r),
                           _ptr(b.select_idx), _ptr(b.select_num), float(scale), _ptr(b.o_r), _ptr(b.o),
                           _ptr(b.ws), b.ws.numel() * b.ws.element_size(), _stream(stream)), "rf_forward")
    return b.o


_PIPELINES = {}        # host pipelines (with their device buffers) of recent problem shapes
_PIPELINES_KEPT = 4


def rainfusion_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         seqs: Sequence[Tuple[int, int, int, int]], sparsity: float = 0.8,
                         layout: str = "BNSD", scale: Optional[float] = None,
                         plan: Optional[Plan] = None, bufs: Optional[Buffers] = None,
                         order: str = "tile", precision: str = "native",
                         chunks: Optional[int] = None, check: bool = True,
                         block_kv: int = 128) -> torch.Tensor:
    """User-level call: RainFusion v2 block-sparse attention of q, k, v (original token order).

    q, k, v may live on the host (pinned or not) or on the GPU; the result is
    returned on the device the inputs came from.  BNSD: q [B, N1, L, D],
    k/v [B, N2, L, D]; TND: q [T, N1, D], k/v [T, N2, D].  `seqs` holds one
    (prefix_len, t, h, w) per sequence (BNSD: one for the whole batch).
    `order` is the token order of the aligned video ("tile", or "frame_pair"
    for 2x8x8 blocks over frame pairs) and `precision` the kernel precision
    ("native", "mix" for E4M3 Q K^T, "fp8" for E4M3 Q K^T and P V, or "mxfp4"
    for MXFP4 attention with UOS scaling and PNQ), and `block_kv` the key block
    length (128, or 64 for aclnnRainFusionAttention's blockShape 128 x 64, whose
    selection ranks 64-row key blocks; native precision); all three are ignored
    when `plan` is given.

    Host inputs run through `pipeline.HostPipeline` (made once per problem
    shape and kept): head chunks whose copies to and from the GPU overlap
    the compute of other chunks; `chunks` overrides its default.  The result
    is the same, bit for bit, as one pass over all heads.

    With check=True (the default) the call then synchronises and reads the
    kernels' status words (aclnnRainFusionAttention returns a status code; a
    CUDA kernel can only record one): an out-of-range selectIdx entry or an
    expired bounded wait raises RfError with status RF_ERR_DEVICE_FAULT, and
    the words are cleared, so the next call starts clean.  check=False skips
    the synchronisation (timing loops); a later call with check=True, or
    check_device_status, still sees what was recorded.
    """
    dtype = {torch.bfloat16: "bf16", torch.float16: "fp16"}[q.dtype]
    if not q.is_cuda and plan is None and bufs is None:
        from .pipeline import HostPipeline
        if layout == "BNSD":
            n1, n2, d, batch = q.shape[1], k.shape[1], q.shape[3], q.shape[0]
        else:
            n1, n2, d, batch = q.shape[1], k.shape[1], q.shape[2], 1
        dev = torch.device("cuda", torch.cuda.current_device())
        key = (tuple(map(tuple, seqs)), n1, n2, d, layout, dtype, float(sparsity), batch, order, precision,
               chunks, dev.index, block_kv)
        pipe = _PIPELINES.pop(key, None)
        if pipe is None:
            pipe = HostPipeline(seqs, n1, n2, d, layout, dtype, sparsity, batch, chunks, order, precision, dev,
                                block_kv)
            while len(_PIPELINES) >= _PIPELINES_KEPT:      # drop the least recently used shape
                _PIPELINES.pop(next(iter(_PIPELINES)))
        _PIPELINES[key] = pipe                               # most recently used last
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        pipe(q, k, v, out, scale)
        torch.cuda.current_stream(dev).synchronize()
        if check:
            pipe.raise_on_device_fault()
        return out
    if plan is None:
        if layout == "BNSD":
            plan = Plan(seqs, q.shape[1], k.shape[1], q.shape[3], "BNSD", dtype, sparsity, batch=q.shape[0],
                        order=order, precision=precision, block_kv=block_kv)
        else:
            plan = Plan(seqs, q.shape[1], k.shape[1], q.shape[2], "TND", dtype, sparsity, order=order,
                        precision=precision, block_kv=block_kv)
    host = not q.is_cuda
    dev = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    if bufs is None:
        bufs = Buffers(plan, dev)
    qd, kd, vd = (x.to(dev, non_blocking=True) for x in (q, k, v))
    out = forward(plan, qd.contiguous(), kd.contiguous(), vd.contiguous(), bufs, scale)
    if check:
        raise_on_device_fault(plan, bufs.ws, "rainfusion_attention")
    if host:
        res = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        res.copy_(out, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        return res
    return out
