"""Top-p routed block-sparse attention forward for NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libfvattn.so`` (C ABI in ``include/fvattn.h``).  The
functions carry the C names; they only marshal arguments: every step of the
computation runs in the library's CUDA kernels.  PyTorch provides device
memory and streams.  There is no CPU fallback: if the library is missing or no
sm_100 device is present, calls raise.

What is computed (page title, section):
  * FVAttn review, §1 Key Terms "Top-p routing": each query block keeps key
    blocks by importance until their cumulative probability reaches p.  The
    score is fixed by this library as mean-pooled blocks, qbar.kbar/sqrt(d),
    softmax over key blocks, ties to the lower index.
  * FlashAttention review, §Model: exact attention as one fused kernel with
    tiled matmuls and tiled online softmax, here restricted to the selected
    key blocks.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfvattn.so")

FVATTN_OK = 0
FVATTN_ERR_INVALID_ARG = -1
FVATTN_ERR_UNSUPPORTED = -2
FVATTN_ERR_ALIGNMENT = -3
FVATTN_ERR_CAPACITY = -4
FVATTN_ERR_CUDA = -5
FVATTN_ERR_BAD_CSR = -6
FVATTN_ERR_DEVICE_TIMEOUT = -7

_lib = None


class FvattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == FVATTN_ERR_CUDA:
            try:
                detail = ": " + load_library().fvattn_last_error().decode()
            except Exception:
                pass
        super().__init__(f"{where}: {status} ({status_string(status)}{detail})")


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libfvattn.so (built in-tree by ``top_routed_block_b200._build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise FvattnError(FVATTN_ERR_UNSUPPORTED, f"libfvattn.so not built (expected at {path}); "
                          "run python -m top_routed_block_b200._build")
    lib = ctypes.CDLL(path)
    P, I, I64, SZ, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_double
    sig = {
        "fvattn_status_string": (ctypes.c_char_p, [I]),
        "fvattn_build_info": (ctypes.c_char_p, []),
        "fvattn_last_error": (ctypes.c_char_p, []),
        "fvattn_num_rows": (I64, [I, I, I, I]),
        "fvattn_route_max_nnz": (I64, [I, I, I, I]),
        "fvattn_route_workspace_bytes": (SZ, [I, I, I, I, I]),
        "fvattn_fwd_workspace_bytes": (SZ, [I, I, I, I]),
        "fvattn_lpt_workspace_bytes": (SZ, [I64, I]),
        "fvattn_route": (I, [P, P, I, I, I, I, I, D, P, P, I64, P, P, SZ, P, P]),
        "fvattn_lpt_order": (I, [P, I64, I, P, P, SZ, P, P]),
        "fvattn_quant_e4m3": (I, [P, I, I, I, I, I, P, P, P]),
        "fvattn_sparse_fwd": (I, [P, P, P, P, P, I, I, I, I, I, I, P, P, P, SZ, P, P]),
        "fvattn_sparse_fwd_noalloc": (I, [P, P, P, P, P, I, I, I, I, I, I, P, P, P, P]),
        "fvattn_test_sparse_fwd_stall": (I, [P, P, P, P, P, I, I, I, I, I, I, P, P, P, SZ, P, P]),
        "fvattn_sparse_fwd_profiled": (I, [P, P, P, P, P, I, I, I, I, I, I, P, P, P, SZ, P, I, P, P, P]),
        "fvattn_attn_num_items": (I64, [I, I, I, I]),
        "fvattn_attn_work_order": (I, [P, P, I, I, I, I, P, P, SZ, P, P]),
        "fvattn_sasa_workspace_bytes": (SZ, [I, I, I, I, I]),
        "fvattn_rlb_plan": (I, [P, I, I, I, P, P, P, P]),
        "fvattn_route_sasa": (I, [P, P, I, I, I, I, I, D, I, P, P, I64, P, P, P, P, P, P, SZ, P, P]),
        "fvattn_sparse_fwd_fp8": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, SZ, P, P]),
        "fvattn_bwd_workspace_bytes": (SZ, [I, I, I, I]),
        "fvattn_sparse_bwd": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, SZ, P, P]),
        "fvattn_attention_host": (I, [P, P, P, I, I, I, I, I, D, I, P, P, P, P, P, P, P, P, P, I64, P, P, SZ, P, SZ,
                                      P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load_library().fvattn_status_string(int(status)).decode()
    except Exception:  # library missing: still describe the code
        return {0: "ok"}.get(int(status), "error")


def _check(rc: int, where: str) -> None:
    if rc != FVATTN_OK:
        raise FvattnError(rc, where)


def _stream_ptr(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else int(t.data_ptr())


def _shape(Q: torch.Tensor):
    if Q.dim() != 4 or Q.dtype != torch.bfloat16 or not Q.is_cuda or not Q.is_contiguous():
        raise ValueError("expected a contiguous CUDA bf16 tensor [B, H, N, d]")
    return tuple(int(x) for x in Q.shape)


def num_blocks(N: int, block: int) -> int:
    return -(-N // block)


def fvattn_num_rows(B: int, H: int, N: int, block: int) -> int:
    return int(load_library().fvattn_num_rows(B, H, N, block))


def fvattn_route_max_nnz(B: int, H: int, N: int, block: int) -> int:
    return int(load_library().fvattn_route_max_nnz(B, H, N, block))


def fvattn_route_workspace_bytes(B: int, H: int, N: int, d: int, block: int) -> int:
    return int(load_library().fvattn_route_workspace_bytes(B, H, N, d, block))


def fvattn_fwd_workspace_bytes(B: int, H: int, N: int, block: int) -> int:
    return int(load_library().fvattn_fwd_workspace_bytes(B, H, N, block))


def fvattn_lpt_workspace_bytes(rows: int, max_count: int) -> int:
    return int(load_library().fvattn_lpt_workspace_bytes(rows, max_count))


@dataclass
class RouteResult:
    row_ptr: torch.Tensor      # int32 [rows + 1]
    col_idx: torch.Tensor      # int32 [capacity]; the first row_ptr[-1] entries are valid
    head_counts: torch.Tensor  # int32 [B*H]
    dev_status: torch.Tensor   # int32 [1]


def _empty_bytes(n: int, device) -> torch.Tensor:
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


def fvattn_route(Q: torch.Tensor, K: torch.Tensor, p: float, block: int, *, stream=None, out: RouteResult | None = None,
                 workspace: torch.Tensor | None = None) -> RouteResult:
    """Top-p routing of (Q, K) into a CSR block mask (asynchronous on ``stream``)."""
    lib = load_library()
    B, H, N, d = _shape(Q)
    if tuple(K.shape) != (B, H, N, d):
        raise ValueError("Q and K shapes differ")
    dev = Q.device
    rows = B * H * num_blocks(N, block)
    if out is None:
        cap = fvattn_route_max_nnz(B, H, N, block)
        out = RouteResult(torch.empty(rows + 1, dtype=torch.int32, device=dev),
                          torch.empty(max(cap, 1), dtype=torch.int32, device=dev),
                          torch.empty(B * H, dtype=torch.int32, device=dev),
                          torch.zeros(1, dtype=torch.int32, device=dev))
    ws_bytes = fvattn_route_workspace_bytes(B, H, N, d, block)
    if workspace is None:
        workspace = _empty_bytes(ws_bytes, dev)
    rc = lib.fvattn_route(_ptr(Q), _ptr(K), B, H, N, d, block, float(p), _ptr(out.row_ptr), _ptr(out.col_idx),
                          out.col_idx.numel(), _ptr(out.head_counts), _ptr(workspace), workspace.numel(),
                          _ptr(out.dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_route")
    return out


def fvattn_lpt_order(row_ptr: torch.Tensor, max_count: int, *, stream=None, order: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None):
    """Rows by selected-block count descending, equal counts by row id."""
    lib = load_library()
    rows = row_ptr.numel() - 1
    dev = row_ptr.device
    if order is None:
        order = torch.empty(max(rows, 1), dtype=torch.int32, device=dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = _empty_bytes(fvattn_lpt_workspace_bytes(rows, max_count), dev)
    rc = lib.fvattn_lpt_order(_ptr(row_ptr), rows, int(max_count), _ptr(order), _ptr(ws), ws.numel(),
                              _ptr(dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_lpt_order")
    return order[:rows], dev_status


def fvattn_quant_e4m3(X: torch.Tensor, block: int, *, stream=None, out: torch.Tensor | None = None,
                      scale_exp: torch.Tensor | None = None):
    """bf16 [B,H,N,d] -> (e4m3 codes uint8 [B,H,N,d], scale exponents int32 [B,H,nb]);
    value = e4m3 value of the code * 2^exponent."""
    lib = load_library()
    B, H, N, d = _shape(X)
    nb = num_blocks(N, block)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.uint8, device=X.device)
    if scale_exp is None:
        scale_exp = torch.empty((B, H, nb), dtype=torch.int32, device=X.device)
    rc = lib.fvattn_quant_e4m3(_ptr(X), B, H, N, d, int(block), _ptr(out), _ptr(scale_exp), _stream_ptr(stream))
    _check(rc, "fvattn_quant_e4m3")
    return out, scale_exp


def fvattn_sparse_fwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                      block: int, causal: bool = False, *, stream=None, O: torch.Tensor | None = None,
                      LSE: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      dev_status: torch.Tensor | None = None):
    """Exact attention over the CSR block mask; returns (O bf16, LSE fp32, dev_status)."""
    lib = load_library()
    B, H, N, d = _shape(Q)
    for t in (K, V):
        if tuple(t.shape) != (B, H, N, d) or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("K and V must match Q")
    dev = Q.device
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _empty_bytes(fvattn_fwd_workspace_bytes(B, H, N, block), dev)
    rc = lib.fvattn_sparse_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(row_ptr), _ptr(col_idx), B, H, N, d, block,
                               1 if causal else 0, _ptr(O), _ptr(LSE), _ptr(workspace), workspace.numel(),
                               _ptr(dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_sparse_fwd")
    return O, LSE, dev_status


def fvattn_sparse_fwd_profiled(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, row_ptr: torch.Tensor,
                               col_idx: torch.Tensor, block: int, causal: bool = False, *, natural_order: bool = False,
                               stream=None, O: torch.Tensor | None = None, LSE: torch.Tensor | None = None,
                               workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None):
    """fvattn_sparse_fwd plus the per-CTA busy time (ns) of its persistent grid.

    Returns (O, LSE, dev_status, busy_ns) with busy_ns an int64 device tensor of one
    entry per launched CTA; ``natural_order`` takes the rows in index order instead
    of the head-major longest-first queue."""
    lib = load_library()
    B, H, N, d = _shape(Q)
    dev = Q.device
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _empty_bytes(fvattn_fwd_workspace_bytes(B, H, N, block), dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    busy = torch.zeros(sms, dtype=torch.int64, device=dev)
    grid = ctypes.c_int(0)
    rc = lib.fvattn_sparse_fwd_profiled(_ptr(Q), _ptr(K), _ptr(V), _ptr(row_ptr), _ptr(col_idx), B, H, N, d, block,
                                        1 if causal else 0, _ptr(O), _ptr(LSE), _ptr(workspace), workspace.numel(),
                                        _ptr(dev_status), 1 if natural_order else 0, _ptr(busy), ctypes.byref(grid),
                                        _stream_ptr(stream))
    _check(rc, "fvattn_sparse_fwd_profiled")
    return O, LSE, dev_status, busy[: grid.value]


def fvattn_sparse_fwd_fp8(Q8: torch.Tensor, K8: torch.Tensor, V8: torch.Tensor, q_exp: torch.Tensor,
                          k_exp: torch.Tensor, v_exp: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                          block: int, causal: bool = False, *, stream=None, O: torch.Tensor | None = None,
                          LSE: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                          dev_status: torch.Tensor | None = None):
    """Block-sparse attention on e4m3 operands (codes uint8 [B,H,N,d] and int32 block
    exponents [B,H,nb], as fvattn_quant_e4m3 returns them).  Returns (O, LSE, dev_status)."""
    lib = load_library()
    B, H, N, d = (int(x) for x in Q8.shape)
    dev = Q8.device
    if O is None:
        O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    if LSE is None:
        LSE = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _empty_bytes(fvattn_fwd_workspace_bytes(B, H, N, block), dev)
    rc = lib.fvattn_sparse_fwd_fp8(_ptr(Q8), _ptr(K8), _ptr(V8), _ptr(q_exp), _ptr(k_exp), _ptr(v_exp), _ptr(row_ptr),
                                   _ptr(col_idx), B, H, N, d, block, 1 if causal else 0, _ptr(O), _ptr(LSE),
                                   _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_sparse_fwd_fp8")
    return O, LSE, dev_status


def fvattn_rlb_plan(work, max_moves: int | None = None):
    """Run-time load balancing moves for per-rank unit work (int [ranks, units], host):
    returns a list of (home unit index, source rank, destination rank)."""
    import numpy as np
    w = np.ascontiguousarray(np.asarray(work), dtype=np.int64)
    ranks, units = (int(x) for x in w.shape)
    cap = 4 * ranks * units + 16 if max_moves is None else int(max_moves)
    mu = np.empty(max(cap, 1), np.int32)
    ms = np.empty(max(cap, 1), np.int32)
    md = np.empty(max(cap, 1), np.int32)
    n = ctypes.c_int32(0)
    rc = load_library().fvattn_rlb_plan(w.ctypes.data, ranks, units, cap, mu.ctypes.data, ms.ctypes.data,
                                        md.ctypes.data, ctypes.byref(n))
    _check(rc, "fvattn_rlb_plan")
    return [(int(mu[k]), int(ms[k]), int(md[k])) for k in range(n.value)]


class SasaResult:
    """Augmented CSR mask, per-head block counts, and per row the number and routing
    probability of the blocks added."""

    def __init__(self, row_ptr, col_idx, head_counts, added, added_mass, dev_status):
        self.row_ptr, self.col_idx, self.head_counts = row_ptr, col_idx, head_counts
        self.added, self.added_mass, self.dev_status = added, added_mass, dev_status


def fvattn_route_sasa(Q: torch.Tensor, K: torch.Tensor, p: float, block: int, machines: int | None = None, *,
                      stream=None, out: SasaResult | None = None, workspace: torch.Tensor | None = None,
                      candidates: bool = False) -> SasaResult:
    """Top-p routing plus slack-aware augmentation over `machines` SMs (default: the
    device's SM count).  With ``candidates``, the result also carries the routing
    candidates (``cand`` int32 and ``cand_p`` fp64, [rows, 8])."""
    lib = load_library()
    B, H, N, d = _shape(Q)
    dev = Q.device
    if machines is None:
        machines = torch.cuda.get_device_properties(dev).multi_processor_count
    rows = fvattn_num_rows(B, H, N, block)
    if out is None:
        cap = fvattn_route_max_nnz(B, H, N, block)
        out = SasaResult(torch.empty(rows + 1, dtype=torch.int32, device=dev),
                         torch.empty(max(cap, 1), dtype=torch.int32, device=dev),
                         torch.empty(B * H, dtype=torch.int32, device=dev),
                         torch.empty(rows, dtype=torch.int32, device=dev),
                         torch.empty(rows, dtype=torch.float64, device=dev),
                         torch.zeros(1, dtype=torch.int32, device=dev))
    out.cand = torch.empty((rows, 8), dtype=torch.int32, device=dev) if candidates else None
    out.cand_p = torch.empty((rows, 8), dtype=torch.float64, device=dev) if candidates else None
    if workspace is None:
        workspace = _empty_bytes(int(lib.fvattn_sasa_workspace_bytes(B, H, N, d, block)), dev)
    rc = lib.fvattn_route_sasa(_ptr(Q), _ptr(K), B, H, N, d, block, float(p), int(machines), _ptr(out.row_ptr),
                               _ptr(out.col_idx), out.col_idx.numel(), _ptr(out.head_counts), _ptr(out.added),
                               _ptr(out.added_mass), _ptr(out.cand), _ptr(out.cand_p), _ptr(workspace),
                               workspace.numel(), _ptr(out.dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_route_sasa")
    return out


def fvattn_attn_num_items(B: int, H: int, N: int, block: int) -> int:
    """Work items of fvattn_sparse_fwd: query blocks at block 128, pairs of them at 64."""
    return int(load_library().fvattn_attn_num_items(B, H, N, block))


def fvattn_attn_work_order(row_ptr: torch.Tensor, B: int, H: int, N: int, block: int,
                           col_idx: torch.Tensor | None = None, *, stream=None, order: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None):
    """The queue order of fvattn_sparse_fwd's work items (item ids: CSR rows at block
    128, pairs of rows 2i, 2i+1 at block 64, which needs col_idx).  Returns the order
    and the device status (FVATTN_ERR_BAD_CSR for a malformed row at block 64)."""
    lib = load_library()
    dev = row_ptr.device
    items = fvattn_attn_num_items(B, H, N, block)
    if order is None:
        order = torch.empty(items, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _empty_bytes(fvattn_fwd_workspace_bytes(B, H, N, block), dev)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = lib.fvattn_attn_work_order(_ptr(row_ptr), _ptr(col_idx), B, H, N, block, _ptr(order), _ptr(workspace),
                                    workspace.numel(), _ptr(dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_attn_work_order")
    return order, dev_status


def fvattn_bwd_workspace_bytes(B: int, H: int, N: int, block: int) -> int:
    return int(load_library().fvattn_bwd_workspace_bytes(B, H, N, block))


def fvattn_sparse_bwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor, LSE: torch.Tensor,
                      dO: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor, block: int,
                      causal: bool = False, *, stream=None, dQ: torch.Tensor | None = None,
                      dK: torch.Tensor | None = None, dV: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None):
    """Gradients of the block-sparse attention; returns (dQ, dK, dV bf16, dev_status)."""
    lib = load_library()
    B, H, N, d = _shape(Q)
    for t in (K, V, O, dO):
        if tuple(t.shape) != (B, H, N, d) or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("K, V, O and dO must match Q")
    dev = Q.device
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(Q) if dK is None else dK
    dV = torch.empty_like(Q) if dV is None else dV
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _empty_bytes(fvattn_bwd_workspace_bytes(B, H, N, block), dev)
    rc = lib.fvattn_sparse_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(dO), _ptr(row_ptr), _ptr(col_idx),
                               B, H, N, d, block, 1 if causal else 0, _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace),
                               workspace.numel(), _ptr(dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_sparse_bwd")
    return dQ, dK, dV, dev_status


def fvattn_sparse_fwd_noalloc(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, row_ptr: torch.Tensor,
                              col_idx: torch.Tensor, block: int, causal: bool, *, O: torch.Tensor, LSE: torch.Tensor,
                              dev_status: torch.Tensor, stream=None):
    """fvattn_sparse_fwd with the library's own fixed device scratch instead of a
    caller workspace; O, LSE and dev_status must be given (nothing is allocated)."""
    lib = load_library()
    B, H, N, d = _shape(Q)
    rc = lib.fvattn_sparse_fwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(row_ptr), _ptr(col_idx), B, H, N, d, block,
                                       1 if causal else 0, _ptr(O), _ptr(LSE), _ptr(dev_status), _stream_ptr(stream))
    _check(rc, "fvattn_sparse_fwd_noalloc")
    return O, LSE, dev_status


def check_status(dev_status: torch.Tensor, where: str = "device") -> None:
    """Synchronise and raise if a kernel recorded an error."""
    torch.cuda.synchronize(dev_status.device)
    for v in dev_status.cpu().tolist():
        _check(int(v), where)


class FvattnPlan:
    """Preallocated device buffers for repeated calls at one shape."""

    def __init__(self, B: int, H: int, N: int, d: int, block: int, device="cuda"):
        self.B, self.H, self.N, self.d, self.block = B, H, N, d, block
        dev = torch.device(device)
        self.device = dev
        self.rows = B * H * num_blocks(N, block)
        self.capacity = fvattn_route_max_nnz(B, H, N, block)
        self.route = RouteResult(torch.empty(self.rows + 1, dtype=torch.int32, device=dev),
                                 torch.empty(max(self.capacity, 1), dtype=torch.int32, device=dev),
                                 torch.empty(B * H, dtype=torch.int32, device=dev),
                                 torch.zeros(1, dtype=torch.int32, device=dev))
        self.route_ws = _empty_bytes(fvattn_route_workspace_bytes(B, H, N, d, block), dev)
        self.fwd_ws = _empty_bytes(fvattn_fwd_workspace_bytes(B, H, N, block), dev)
        self.O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
        self.LSE = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.status = torch.zeros(3, dtype=torch.int32, device=dev)   # route, attention, first error (host path)

    def run_route(self, Q, K, p, stream=None) -> RouteResult:
        return fvattn_route(Q, K, p, self.block, stream=stream, out=self.route, workspace=self.route_ws)

    def run_fwd(self, Q, K, V, causal=False, row_ptr=None, col_idx=None, stream=None):
        rp = self.route.row_ptr if row_ptr is None else row_ptr
        ci = self.route.col_idx if col_idx is None else col_idx
        return fvattn_sparse_fwd(Q, K, V, rp, ci, self.block, causal, stream=stream, O=self.O, LSE=self.LSE,
                                 workspace=self.fwd_ws, dev_status=self.status[1:])

    def __call__(self, Q, K, V, p, causal=False, stream=None):
        self.run_route(Q, K, p, stream=stream)
        return self.run_fwd(Q, K, V, causal, stream=stream)

    def check(self):
        self.status[0:1].copy_(self.route.dev_status)
        check_status(self.status[:2], "fvattn")


def fvattn_attention_host(hQ: torch.Tensor, hK: torch.Tensor, hV: torch.Tensor, p: float, block: int,
                          causal: bool = False, *, plan: FvattnPlan, dQ: torch.Tensor, dK: torch.Tensor,
                          dV: torch.Tensor, hO: torch.Tensor, hLSE: torch.Tensor, stream=None) -> None:
    """Whole path from host buffers: H2D copies, routing, sparse forward, D2H copies (synchronous)."""
    lib = load_library()
    B, H, N, d = (int(x) for x in hQ.shape)
    pl = plan
    rc = lib.fvattn_attention_host(_ptr(hQ), _ptr(hK), _ptr(hV), B, H, N, d, block, float(p), 1 if causal else 0,
                                   _ptr(hO), _ptr(hLSE), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(pl.O), _ptr(pl.LSE),
                                   _ptr(pl.route.row_ptr), _ptr(pl.route.col_idx), pl.route.col_idx.numel(),
                                   _ptr(pl.route.head_counts), _ptr(pl.route_ws), pl.route_ws.numel(), _ptr(pl.fwd_ws),
                                   pl.fwd_ws.numel(), _ptr(pl.status), _stream_ptr(stream))
    _check(rc, "fvattn_attention_host")


__all__ = [n for n in dir() if n.startswith("fvattn_")] + ["FvattnPlan", "FvattnError", "RouteResult",
                                                          "check_status", "load_library", "status_string"]
