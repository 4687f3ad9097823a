"""Python binding of libbsa.so (include/bsa.h): argument marshalling only.

Every call here converts torch tensors to device pointers and forwards to the
C ABI of the same name; all computation runs in the library's CUDA kernels.
There is no CPU path: tensors must live on a CUDA device, and importing the
binding without the built library raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbsa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE, ERR_INFEASIBLE = range(7)
DEVERR_NONE, DEVERR_BAD_INDEX, DEVERR_TIMEOUT, DEVERR_SCHEDULE, DEVERR_NO_GEOMETRY = range(5)
HEAD_FULL, HEAD_SPARSE, HEAD_SKIP = 0, 1, 2
BLOCK_NONE, BLOCK_FULL, BLOCK_PARTIAL = 0, 1, 2
MASK_ARROW, MASK_GNA = 1, 2
SELECT_POOLED_QK, SELECT_FULL_SCORE = 1, 2
STEP_FULL, STEP_SELECT, STEP_REUSE = 0, 1, 2

EXPORTS = (
    "bsa_version", "bsa_error_string", "bsa_build_mask", "bsa_select_workspace_size",
    "bsa_select_topk", "bsa_forward", "bsa_gna_tiled_len", "bsa_permute_tiles",
    "bsa_unpermute_tiles", "bsa_get_device_error", "bsa_select_topk_static", "bsa_rse",
    "bsa_plan_heads", "bsa_schedule_full_steps", "bsa_step_action", "bsa_keep_pct", "bsa_jaccard",
    "bsa_set_wait_limit_ns", "bsa_set_withheld_tile", "bsa_quantize_fp8", "bsa_forward_fp8",
)
STATIC_SCRATCH_BYTES = 16 << 20


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib().bsa_error_string(status).decode()} (status {status})")


# ---------------------------------------------------------------------------- structs

class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
                ("n_text", ctypes.c_int32)]


class GnaGeom(ctypes.Structure):
    _fields_ = [("ndim", ctypes.c_int32), ("grid", ctypes.c_int32 * 3), ("tile", ctypes.c_int32 * 3),
                ("window", ctypes.c_int32 * 3), ("stride", ctypes.c_int32 * 3)]

    @classmethod
    def make(cls, grid, tile, window, stride):
        n = len(grid)
        g = cls()
        g.ndim = n
        for i in range(n):
            g.grid[i], g.tile[i], g.window[i], g.stride[i] = grid[i], tile[i], window[i], stride[i]
        return g


class MaskSpec(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("head_mode", ctypes.c_void_p), ("window", ctypes.c_void_p),
                ("gna", GnaGeom)]


class BlockListC(ctypes.Structure):
    _fields_ = [("cnt", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("flag", ctypes.c_void_p),
                ("bitmap", ctypes.c_void_p), ("max_k", ctypes.c_int32)]


class KeyGroup(ctypes.Structure):
    _fields_ = [("begin", ctypes.c_int32), ("end", ctypes.c_int32), ("k", ctypes.c_int32)]


class SelectSpec(ctypes.Structure):
    _fields_ = [("method", ctypes.c_int32), ("n_groups", ctypes.c_int32), ("groups", KeyGroup * 4),
                ("keep_text", ctypes.c_int32), ("scale", ctypes.c_float)]


# ---------------------------------------------------------------------------- library

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libbsa.so not built at {LIB_PATH}: run "
                              "python -m block_sparse_attention_37_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        lib.bsa_version.restype = ctypes.c_int
        lib.bsa_error_string.restype = ctypes.c_char_p
        lib.bsa_error_string.argtypes = [ctypes.c_int]
        lib.bsa_build_mask.argtypes = [P, P, P, P]
        lib.bsa_select_workspace_size.restype = ctypes.c_size_t
        lib.bsa_select_workspace_size.argtypes = [P, P]
        lib.bsa_select_topk.argtypes = [P, P, P, P, P, P, ctypes.c_size_t, P, P]
        lib.bsa_forward.argtypes = [P, P, P, P, P, P, P, P, P, P, ctypes.c_float, P, P]
        lib.bsa_gna_tiled_len.argtypes = [ctypes.c_int32, P, P]
        lib.bsa_permute_tiles.argtypes = [P, P, ctypes.c_int32, P, P, P]
        lib.bsa_unpermute_tiles.argtypes = [P, P, ctypes.c_int32, P, P, P]
        lib.bsa_get_device_error.argtypes = [P, P]
        lib.bsa_select_topk_static.argtypes = [P, P, P, P, P, P, P]
        lib.bsa_rse.argtypes = [P, P, P, P, P]
        lib.bsa_plan_heads.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_double, ctypes.c_double,
                                       P, P]
        I32 = ctypes.c_int32
        lib.bsa_schedule_full_steps.argtypes = [I32, I32, P]
        lib.bsa_step_action.argtypes = [I32, I32, I32, P]
        lib.bsa_keep_pct.argtypes = [I32, I32, I32, I32, I32, I32, P]
        lib.bsa_jaccard.argtypes = [P, P, P, P, P]
        lib.bsa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.bsa_quantize_fp8.argtypes = [P] * 11
        lib.bsa_forward_fp8.argtypes = [P] * 13 + [ctypes.c_float, P, P]
        lib.bsa_set_withheld_tile.argtypes = [I32]
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes library (raises ImportError if it was not built)."""
    return _lib()


def _check(status: int, where: str):
    if status != OK:
        raise BsaError(status, where)


def _check_buffer(t, dtype=None, name="tensor", numel=None):
    """Type, dtype and size of `t` (None passes). The library reads and writes
    through raw pointers, so a buffer smaller than the layout the header states
    would be accessed out of bounds: refuse it here."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; these dims need {numel}")


def _ptr(t, dtype=None, name="tensor", numel=None):
    """Device pointer of `t` after the buffer check and the device checks."""
    if t is None:
        return None
    _check_buffer(t, dtype, name, numel)
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _ptrs(*specs):
    """Pointers for (tensor, dtype, name, numel) specs. Every type and size is
    checked before any device check, so a wrong size is reported as such."""
    for sp in specs:
        _check_buffer(*sp)
    return [_ptr(*sp) for sp in specs]


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def version() -> int:
    """Library version, major*10000 + minor*100 + patch (bsa_version)."""
    return _lib().bsa_version()


def dims(B, H, N, d, block_q, block_k, n_text) -> Dims:
    """Problem shape (bsa_dims): batch, heads, tokens, head dim, query / key block sizes, text tokens."""
    return Dims(B, H, N, d, block_q, block_k, n_text)


def n_blocks(n: int, bs: int) -> int:
    """ceil(n / bs): blocks of size bs over n tokens (the last one ragged)."""
    return -(-n // bs)


def _tokens(dm: Dims) -> int:
    """Elements of one [B, H, N, d] tensor."""
    return max(dm.B, 0) * max(dm.H, 0) * max(dm.N, 0) * max(dm.d, 0)


def _grid(dm: Dims):
    """(rows, nQB, nKB) of the block lists and bitmaps for these dims."""
    nQB = n_blocks(dm.N, dm.block_q) if dm.block_q > 0 else 0
    nKB = n_blocks(dm.N, dm.block_k) if dm.block_k > 0 else 0
    return max(dm.B, 0) * max(dm.H, 0) * nQB, nQB, nKB


@dataclass
class BlockList:
    """Device buffers of a block list (see bsa_block_list)."""
    cnt: torch.Tensor
    idx: torch.Tensor
    flag: torch.Tensor
    bitmap: torch.Tensor | None
    max_k: int

    @classmethod
    def empty(cls, B, H, nQB, nKB, max_k=None, device="cuda", bitmap=True):
        max_k = nKB if max_k is None else max_k
        return cls(
            cnt=torch.empty((B, H, nQB), dtype=torch.int32, device=device),
            idx=torch.empty((B, H, nQB, max_k), dtype=torch.int32, device=device),
            flag=torch.empty((B, H, nQB, max_k), dtype=torch.uint8, device=device),
            bitmap=torch.empty((B, H, nQB, nKB), dtype=torch.uint8, device=device) if bitmap else None,
            max_k=max_k)

    def specs(self, dm: Dims | None = None):
        """Buffer specs of cnt, idx, flag and bitmap; with `dm`, each must hold
        its [B, H, nQB(, max_k | nKB)] layout."""
        rows, _, nKB = _grid(dm) if dm is not None else (None, 0, 0)
        need = (lambda w: rows * w) if dm is not None else (lambda w: None)
        return [(self.cnt, torch.int32, "cnt", need(1)), (self.idx, torch.int32, "idx", need(self.max_k)),
                (self.flag, torch.uint8, "flag", need(self.max_k)),
                (self.bitmap, torch.uint8, "bitmap", need(nKB))]

    def c(self, dm: Dims | None = None, ptrs=None) -> BlockListC:
        """The C struct (from already checked pointers, if given)."""
        p = _ptrs(*self.specs(dm)) if ptrs is None else ptrs
        return BlockListC(*p, self.max_k)


# ---------------------------------------------------------------------------- calls

def build_mask(dm: Dims, kind: int, out: BlockList, head_mode=None, window=None, gna: GnaGeom | None = None,
               stream=None):
    """bsa_build_mask: arrow (MASK_ARROW, window per head in blocks) or GNA (MASK_GNA, tile-order
    tokens, block = tile volume) block lists into `out` for every (b, h, query block).
    head_mode / window: cuda int32 [H] (head_mode None = all SPARSE)."""
    p = _ptrs(*out.specs(dm), (head_mode, torch.int32, "head_mode", dm.H), (window, torch.int32, "window", dm.H))
    spec = MaskSpec(kind, p[4], p[5], gna if gna is not None else GnaGeom())
    lc = out.c(dm, p[:4])
    _check(_lib().bsa_build_mask(ctypes.byref(dm), ctypes.byref(spec), ctypes.byref(lc), _stream(stream)),
           "bsa_build_mask")


def select_spec(method: int, groups, keep_text: bool, scale: float = 1.0) -> SelectSpec:
    """Selection spec: method (SELECT_POOLED_QK / SELECT_FULL_SCORE), up to four (begin, end, k) key
    block groups each cut to its own top k, whether text blocks are always kept, the logit scale."""
    sp = SelectSpec()
    sp.method = method
    sp.n_groups = len(groups)
    for i, (b, e, k) in enumerate(groups):
        sp.groups[i] = KeyGroup(b, e, k)
    sp.keep_text = 1 if keep_text else 0
    sp.scale = scale
    return sp


def select_workspace_size(dm: Dims, spec: SelectSpec) -> int:
    """Bytes of device workspace bsa_select_topk needs for these dims and spec."""
    return int(_lib().bsa_select_workspace_size(ctypes.byref(dm), ctypes.byref(spec)))


def select_topk(dm: Dims, q, k, spec: SelectSpec, out: BlockList, workspace, bias=None, stream=None):
    """bsa_select_topk: content-driven block lists into `out`. q, k: cuda bf16 [B, H, N, d];
    workspace: cuda tensor of at least select_workspace_size bytes, 256-byte aligned;
    bias: cuda fp32 [H, nQB, nKB] logit offset (FULL_SCORE) or None."""
    n, (_, nQB, nKB) = _tokens(dm), _grid(dm)
    p = _ptrs(*out.specs(dm), (q, torch.bfloat16, "Q", n), (k, torch.bfloat16, "K", n),
              (bias, torch.float32, "bias", dm.H * nQB * nKB), (workspace, None, "workspace", None))
    lc = out.c(dm, p[:4])
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib().bsa_select_topk(ctypes.byref(dm), p[4], p[5], ctypes.byref(spec), p[6], p[7], ws_bytes,
                                  ctypes.byref(lc), _stream(stream)), "bsa_select_topk")


def select_topk_static(dm: Dims, q, k, spec: SelectSpec, out: BlockList, bias=None, stream=None):
    """bsa_select_topk_static: selection with the library's fixed scratch (no allocation)."""
    n, (_, nQB, nKB) = _tokens(dm), _grid(dm)
    p = _ptrs(*out.specs(dm), (q, torch.bfloat16, "Q", n), (k, torch.bfloat16, "K", n),
              (bias, torch.float32, "bias", dm.H * nQB * nKB))
    lc = out.c(dm, p[:4])
    _check(_lib().bsa_select_topk_static(ctypes.byref(dm), p[4], p[5], ctypes.byref(spec), p[6], ctypes.byref(lc),
                                         _stream(stream)),
           "bsa_select_topk_static")


def forward(dm: Dims, q, k, v, o, head_mode, blocks: BlockList | None = None, gna: GnaGeom | None = None,
            cache_in=None, cache_out=None, bias=None, scale: float | None = None, stream=None):
    """bsa_forward: o (cuda bf16 [B, H, N, d]) = block-sparse attention of q, k, v (same shape) over
    the kept blocks; per head FULL / SPARSE (the block list) / SKIP (o = bf16 of cache_in, fp32
    [B, H, N, d]). cache_out receives the fp32 output of computed heads; bias is a cuda fp32
    [H, nQB, nKB] logit offset; scale defaults to 1/sqrt(d); gna is needed for PARTIAL blocks."""
    scale = (1.0 / dm.d ** 0.5) if scale is None else scale
    n, (_, nQB, nKB) = _tokens(dm), _grid(dm)
    ls = blocks.specs(dm) if blocks is not None else []
    p = _ptrs(*ls, (q, torch.bfloat16, "Q", n), (k, torch.bfloat16, "K", n), (v, torch.bfloat16, "V", n),
              (o, torch.bfloat16, "O", n), (head_mode, torch.int32, "head_mode", dm.H),
              (cache_in, torch.float32, "cache_in", n), (cache_out, torch.float32, "cache_out", n),
              (bias, torch.float32, "bias", dm.H * nQB * nKB))
    lc = blocks.c(dm, p[:4]) if blocks is not None else None
    qp, kp, vp, op, hm, ci, co, bp = p[len(ls):]
    _check(_lib().bsa_forward(ctypes.byref(dm), qp, kp, vp, ctypes.byref(lc) if lc is not None else None, hm,
                              ctypes.byref(gna) if gna is not None else None, ci, co, bp, float(scale), op,
                              _stream(stream)), "bsa_forward")


@dataclass
class Fp8Operands:
    """The e4m3 operands bsa_quantize_fp8 writes: codes of Q and K (uint8 [B, H, N, 128]), V's
    codes transposed per head (uint8 [B, H, 128, Nt], Nt = N rounded up to 16) and the fp32
    scales per 64-token block ([B, H, ceil(N / 64)])."""
    q8: torch.Tensor
    k8: torch.Tensor
    v8t: torch.Tensor
    sq: torch.Tensor
    sk: torch.Tensor
    sv: torch.Tensor

    @staticmethod
    def empty(B: int, H: int, N: int, d: int = 128, device="cuda") -> "Fp8Operands":
        nt, ns = (N + 15) // 16 * 16, n_blocks(N, 64)
        u8 = lambda *shape: torch.empty(shape, dtype=torch.uint8, device=device)
        f32 = lambda: torch.empty((B, H, ns), dtype=torch.float32, device=device)
        return Fp8Operands(u8(B, H, N, d), u8(B, H, N, d), u8(B, H, d, nt), f32(), f32(), f32())

    def specs(self, dm: Dims):
        n, nt, ns = _tokens(dm), (dm.N + 15) // 16 * 16, n_blocks(dm.N, 64)
        bh = max(dm.B, 0) * max(dm.H, 0)
        return [(self.q8, torch.uint8, "q8", n), (self.k8, torch.uint8, "k8", n),
                (self.v8t, torch.uint8, "v8t", bh * dm.d * nt), (self.sq, torch.float32, "sq", bh * ns),
                (self.sk, torch.float32, "sk", bh * ns), (self.sv, torch.float32, "sv", bh * ns)]


def quantize_fp8(dm: Dims, q, k, v, ops: Fp8Operands, stream=None):
    """bsa_quantize_fp8: e4m3 codes and per-64-token-block scales of q, k, v (cuda bf16
    [B, H, N, 128]) into `ops` (Fp8Operands.empty(B, H, N))."""
    n = _tokens(dm)
    p = _ptrs((q, torch.bfloat16, "Q", n), (k, torch.bfloat16, "K", n), (v, torch.bfloat16, "V", n),
              *ops.specs(dm))
    _check(_lib().bsa_quantize_fp8(ctypes.byref(dm), *p, _stream(stream)), "bsa_quantize_fp8")


def forward_fp8(dm: Dims, ops: Fp8Operands, o, head_mode, blocks: BlockList | None = None,
                gna: GnaGeom | None = None, cache_in=None, cache_out=None, bias=None, scale: float | None = None,
                stream=None):
    """bsa_forward_fp8: bsa_forward on the e4m3 operands of quantize_fp8; o is cuda bf16 [B, H, N, 128]."""
    scale = (1.0 / dm.d ** 0.5) if scale is None else scale
    n, (_, nQB, nKB) = _tokens(dm), _grid(dm)
    ls = blocks.specs(dm) if blocks is not None else []
    p = _ptrs(*ls, *ops.specs(dm), (o, torch.bfloat16, "O", n), (head_mode, torch.int32, "head_mode", dm.H),
              (cache_in, torch.float32, "cache_in", n), (cache_out, torch.float32, "cache_out", n),
              (bias, torch.float32, "bias", dm.H * nQB * nKB))
    lc = blocks.c(dm, p[:4]) if blocks is not None else None
    q8, k8, v8t, sq, sk, sv, op, hm, ci, co, bp = p[len(ls):]
    _check(_lib().bsa_forward_fp8(ctypes.byref(dm), q8, k8, v8t, sq, sk, sv,
                                  ctypes.byref(lc) if lc is not None else None, hm,
                                  ctypes.byref(gna) if gna is not None else None, ci, co, bp, float(scale), op,
                                  _stream(stream)), "bsa_forward_fp8")


def gna_tiled_len(n_text: int, gna: GnaGeom) -> int:
    """Tokens in tile order: text padded to a tile-volume multiple plus every (padded) tile."""
    n = ctypes.c_int32(0)
    _check(_lib().bsa_gna_tiled_len(int(n_text), ctypes.byref(gna), ctypes.byref(n)), "bsa_gna_tiled_len")
    return int(n.value)


def _ptr_arrays(ins, n_in, outs, n_out):
    """Host arrays of the device pointers of `ins` and `outs` (bf16, checked)."""
    if len(ins) != len(outs):
        raise ValueError("the permutation needs as many outputs as inputs")
    specs = [(t, torch.bfloat16, f"in[{i}]", n_in) for i, t in enumerate(ins)] + \
            [(t, torch.bfloat16, f"out[{i}]", n_out) for i, t in enumerate(outs)]
    p = _ptrs(*specs)
    a_in, a_out = (ctypes.c_void_p * len(ins))(), (ctypes.c_void_p * len(outs))()
    for i in range(len(ins)):
        a_in[i], a_out[i] = p[i].value, p[len(ins) + i].value
    return a_in, a_out


def _permute_sizes(dm: Dims, gna: GnaGeom):
    """Elements of one raster tensor and of one tile-order tensor."""
    grid = 1
    for i in range(max(0, min(gna.ndim, 3))):
        grid *= gna.grid[i]
    bhd = max(dm.B, 0) * max(dm.H, 0) * max(dm.d, 0)
    return bhd * (dm.n_text + grid), bhd * gna_tiled_len(dm.n_text, gna)


def permute_tiles(dm: Dims, gna: GnaGeom, ins, outs, stream=None):
    """bsa_permute_tiles: raster [B, H, n_text + prod(grid), d] bf16 tensors to tile order
    [B, H, gna_tiled_len, d] (padding rows zeroed), one output per input (at most four)."""
    n_r, n_t = _permute_sizes(dm, gna)
    a_in, a_out = _ptr_arrays(ins, n_r, outs, n_t)
    _check(_lib().bsa_permute_tiles(ctypes.byref(dm), ctypes.byref(gna), len(ins), a_in, a_out, _stream(stream)),
           "bsa_permute_tiles")


def unpermute_tiles(dm: Dims, gna: GnaGeom, ins, outs, stream=None):
    """bsa_unpermute_tiles: the inverse of permute_tiles (padding rows dropped)."""
    n_r, n_t = _permute_sizes(dm, gna)
    a_in, a_out = _ptr_arrays(ins, n_t, outs, n_r)
    _check(_lib().bsa_unpermute_tiles(ctypes.byref(dm), ctypes.byref(gna), len(ins), a_in, a_out, _stream(stream)),
           "bsa_unpermute_tiles")


def rse(dm: Dims, y_m, y_o, out, stream=None):
    """bsa_rse: out (cuda float64 [4*H]) receives I(h) then the three sums per head."""
    n = _tokens(dm)
    p = _ptrs((y_m, torch.bfloat16, "y_m", n), (y_o, torch.bfloat16, "y_o", n),
              (out, torch.float64, "out", 4 * max(dm.H, 0)))
    _check(_lib().bsa_rse(ctypes.byref(dm), *p, _stream(stream)), "bsa_rse")


def plan_heads(rse_hm, cost_hm, delta: float, c: float = 1.5):
    """bsa_plan_heads on host arrays [H, M]; returns (choice int32 [H], total cost)."""
    import numpy as np
    r = np.ascontiguousarray(rse_hm, dtype=np.float64)
    k = np.ascontiguousarray(cost_hm, dtype=np.int64)
    if r.ndim != 2 or r.shape != k.shape:
        raise ValueError("rse and cost must both be [H, M]")
    H, M = r.shape
    choice = np.zeros(H, dtype=np.int32)
    total = ctypes.c_int64(0)
    _check(_lib().bsa_plan_heads(H, M, r.ctypes.data_as(ctypes.c_void_p), k.ctypes.data_as(ctypes.c_void_p),
                                 float(delta), float(c), choice.ctypes.data_as(ctypes.c_void_p),
                                 ctypes.byref(total)), "bsa_plan_heads")
    return choice, int(total.value)


def schedule_full_steps(n_steps: int, skip_pct: int) -> int:
    """bsa_schedule_full_steps (host only)."""
    v = ctypes.c_int32(0)
    _check(_lib().bsa_schedule_full_steps(n_steps, skip_pct, ctypes.byref(v)), "bsa_schedule_full_steps")
    return v.value


def step_action(step: int, n_steps: int, n_full: int) -> int:
    """bsa_step_action (host only): STEP_FULL, STEP_SELECT or STEP_REUSE."""
    v = ctypes.c_int32(0)
    _check(_lib().bsa_step_action(step, n_steps, n_full, ctypes.byref(v)), "bsa_step_action")
    return v.value


def keep_pct(layer: int, n_layers: int, step: int, n_steps: int, hi: int, lo: int) -> int:
    """bsa_keep_pct (host only)."""
    v = ctypes.c_int32(0)
    _check(_lib().bsa_keep_pct(layer, n_layers, step, n_steps, hi, lo, ctypes.byref(v)), "bsa_keep_pct")
    return v.value


def jaccard(dm: Dims, a: BlockList, b: BlockList, out, stream=None):
    """bsa_jaccard: out (cuda float32 [B, H, nQB]) receives the per-row similarity."""
    p = _ptrs(*a.specs(dm), *b.specs(dm), (out, torch.float32, "out", _grid(dm)[0]))
    ca, cb = a.c(dm, p[0:4]), b.c(dm, p[4:8])
    _check(_lib().bsa_jaccard(ctypes.byref(dm), ctypes.byref(ca), ctypes.byref(cb), p[8], _stream(stream)),
           "bsa_jaccard")


def set_wait_limit_ns(ns: int) -> None:
    """Bound of every pipeline wait in later forward / full-score selection launches (0: default 2 s)."""
    _check(_lib().bsa_set_wait_limit_ns(int(ns)), "bsa_set_wait_limit_ns")


def set_withheld_tile(tile: int) -> None:
    """Test hook: later forwards never load this key tile's K, so its waits run out (-1: off)."""
    _check(_lib().bsa_set_withheld_tile(int(tile)), "bsa_set_withheld_tile")


def get_device_error(stream=None) -> int:
    """Synchronise the stream, then read and clear the device error word (a DEVERR_* value)."""
    code = ctypes.c_int32(0)
    _check(_lib().bsa_get_device_error(_stream(stream), ctypes.byref(code)), "bsa_get_device_error")
    return int(code.value)
