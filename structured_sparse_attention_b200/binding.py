"""Thin ctypes binding of libssa (declared in include/ssa.h).

Argument marshalling only: torch provides device memory and the current stream; every
step of the computation runs in the library's CUDA kernels.  There is no fallback: if
libssa.so is missing or no CUDA device is present the calls raise.

A caller-provided ``status`` tensor (one int32 on the device) is used as is: the
caller zeroes it and reads it (the functions read it themselves when ``check``).
"""

from __future__ import annotations

import ctypes as C
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssa.so")

SSA_OK = 0
ERRORS = {-1: "SSA_ERR_INVALID", -2: "SSA_ERR_UNSUPPORTED", -3: "SSA_ERR_CAPACITY",
          -4: "SSA_ERR_CUDA", -5: "SSA_ERR_TIMEOUT"}
BLOCK = 128

#: Every symbol include/ssa.h declares.
EXPORTS = ("sparse_attn_maps", "sparse_pattern_capture_ws_bytes", "sparse_pattern_capture", "sparse_pattern_capture_ex",
           "sparse_pattern_capture_noalloc", "sparse_pattern_extend_case2",
           "sparse_pattern_extend_ws_bytes", "sparse_pattern_extend",
           "sparse_attn_fwd_ws_bytes", "sparse_attn_fwd",
           "sparse_attn_decode_ws_bytes", "sparse_attn_decode",
           "ssa_last_error", "ssa_version", "ssa_set_wait_limit_ns")


class SSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class PlanSizes(C.Structure):
    _fields_ = [("n_heads", C.c_int32), ("S", C.c_int32), ("nqb", C.c_int32),
                ("n_diag", C.c_int32), ("n_vert", C.c_int32), ("max_vert", C.c_int32),
                ("n_tiles", C.c_int64), ("bitmap_slots", C.c_int32)]


class PlanStruct(C.Structure):
    _fields_ = [("n_heads", C.c_int32), ("S", C.c_int32), ("nqb", C.c_int32),
                ("max_vert", C.c_int32), ("n_tiles", C.c_int64),
                ("ext_diag_ptr", C.c_void_p), ("ext_diag_offsets", C.c_void_p),
                ("ext_vert_ptr", C.c_void_p), ("ext_vert_cols", C.c_void_p),
                ("tile_ptr", C.c_void_p), ("tile_key0", C.c_void_p), ("tile_dmask", C.c_void_p),
                ("tile_cmask", C.c_void_p), ("tile_flags", C.c_void_p), ("stripe_cnt", C.c_void_p),
                ("bitmap_slots", C.c_int32), ("tile_bits", C.c_void_p),
                ("n_diag", C.c_int32), ("n_vert", C.c_int32)]


_lib = None


def load():
    """Load libssa.so (built in-tree by ``__graft_entry__.build()``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise SSAError(-4, f"{LIB_PATH} is not built; run __graft_entry__.build()")
        lib = C.CDLL(LIB_PATH)
        V, I, D, SZ = C.c_void_p, C.c_int, C.c_double, C.c_size_t
        lib.sparse_attn_maps.argtypes = [V, V, I, I, I, I, C.c_float, V, V, V]
        lib.sparse_attn_maps.restype = I
        lib.sparse_pattern_capture_ws_bytes.argtypes = [I, I]
        lib.sparse_pattern_capture_ws_bytes.restype = SZ
        lib.sparse_pattern_capture.argtypes = [V, I, I, D, D, D, D, V, V, V, V, V, SZ, V, V]
        lib.sparse_pattern_capture.restype = I
        lib.sparse_pattern_capture_ex.argtypes = [V, I, I, D, D, D, D, I, V, V, V, V, V, V, SZ, V, V]
        lib.sparse_pattern_capture_ex.restype = I
        lib.sparse_pattern_extend_case2.argtypes = [I, V, V, V, V, V, I, I, C.POINTER(PlanSizes),
                                                    C.POINTER(PlanStruct), V, SZ, V, V]
        lib.sparse_pattern_extend_case2.restype = I
        lib.sparse_pattern_extend_ws_bytes.argtypes = [I, I]
        lib.sparse_pattern_extend_ws_bytes.restype = SZ
        lib.sparse_pattern_extend.argtypes = [I, V, V, V, V, I, C.POINTER(PlanSizes),
                                              C.POINTER(PlanStruct), V, SZ, V, V]
        lib.sparse_pattern_extend.restype = I
        lib.sparse_attn_fwd_ws_bytes.argtypes = [I, I, I]
        lib.sparse_attn_fwd_ws_bytes.restype = SZ
        lib.sparse_attn_fwd.argtypes = [V, V, V, I, I, I, I, C.POINTER(PlanStruct), V, C.c_float,
                                        V, V, V, SZ, V, V]
        lib.sparse_attn_fwd.restype = I
        lib.sparse_attn_decode_ws_bytes.argtypes = [I, I, I]
        lib.sparse_attn_decode_ws_bytes.restype = SZ
        lib.sparse_attn_decode.argtypes = [V, V, V, I, I, I, I, I, V, C.POINTER(PlanStruct), V, C.c_float,
                                           V, V, V, SZ, V, V]
        lib.sparse_attn_decode.restype = I
        lib.ssa_last_error.argtypes = []
        lib.ssa_last_error.restype = C.c_char_p
        lib.ssa_version.restype = I
        lib.ssa_set_wait_limit_ns.argtypes = [C.c_int64]
        lib.ssa_set_wait_limit_ns.restype = C.c_int64
        _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream), s


def _check(rc: int):
    if rc != SSA_OK:
        raise SSAError(rc, load().ssa_last_error().decode())


def _check_status(status: torch.Tensor, stream):
    stream.synchronize()
    code = int(status.item())
    if code != 0:
        raise SSAError(code, "reported by a kernel (dev_status)")


def _need_cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise SSAError(-1, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise SSAError(-1, f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise SSAError(-1, f"{name} must have dtype {dtype}, got {t.dtype}")


def set_wait_limit_ns(ns: int) -> int:
    return int(load().ssa_set_wait_limit_ns(int(ns)))


# ------------------------------------------------------------------------------------
# Stage one
# ------------------------------------------------------------------------------------

def attn_maps(q: torch.Tensor, k: torch.Tensor, scale: float = None, *, stream=None, check: bool = True,
              out=None, status=None):
    """sparse_attn_maps: q, k bf16 [n_maps, B, L, d] (CUDA) -> averaged causal attention
    maps float32 [n_maps, L, L] (entries above the diagonal are 0)."""
    lib = load()
    _need_cuda(q, "q", torch.bfloat16)
    _need_cuda(k, "k", torch.bfloat16)
    if q.dim() != 4 or q.shape != k.shape:
        raise SSAError(-1, "q and k must both be [n_maps, B, L, d]")
    n, B, L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((n, L, L), dtype=torch.float32, device=q.device)
    _need_cuda(out, "out", torch.float32)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    cs, s = _stream(stream)
    _check(lib.sparse_attn_maps(_ptr(q), _ptr(k), n, B, L, d, float(scale), _ptr(out), _ptr(status), cs))
    if check:
        _check_status(status, s)
    return out


SCALINGS = {"row": 0, "map": 1}  # SSA_SCALE_ROW, SSA_SCALE_MAP


def capture(maps: torch.Tensor, lam: float = 0.5, tau: float = 0.3, mu: float = 0.8,
            eps: float = 1e-8, *, scaling: str = "row", true_mask: bool = False, stream=None,
            check: bool = True, out=None, ws=None, status=None):
    """sparse_pattern_capture(_ex) on maps [n, L, L] float32 (CUDA).  Returns a dict of CUDA
    int32 tensors: diag_ptr [n+1], diag_offsets [n*L], vert_ptr [n+1], vert_cols [n*L], and
    with true_mask=True also "true_mask": the bitmap uint32 [n, L, ceil(L/32)] (as int32)."""
    lib = load()
    _need_cuda(maps, "maps", torch.float32)
    n, L, L2 = maps.shape
    if L != L2:
        raise SSAError(-1, "maps must be [n, L, L]")
    dev = maps.device
    if out is None:
        out = dict(diag_ptr=torch.empty(n + 1, dtype=torch.int32, device=dev),
                   diag_offsets=torch.empty(max(n * L, 1), dtype=torch.int32, device=dev),
                   vert_ptr=torch.empty(n + 1, dtype=torch.int32, device=dev),
                   vert_cols=torch.empty(max(n * L, 1), dtype=torch.int32, device=dev))
    need = lib.sparse_pattern_capture_ws_bytes(n, L)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    cs, s = _stream(stream)
    if scaling not in SCALINGS:
        raise SSAError(-1, f"scaling must be one of {sorted(SCALINGS)}")
    if true_mask and "true_mask" not in out:
        out["true_mask"] = torch.empty((n, L, (L + 31) // 32), dtype=torch.int32, device=dev)
    if scaling == "row" and not true_mask:
        _check(lib.sparse_pattern_capture(_ptr(maps), n, L, lam, tau, mu, eps, _ptr(out["diag_ptr"]),
                                          _ptr(out["diag_offsets"]), _ptr(out["vert_ptr"]),
                                          _ptr(out["vert_cols"]), _ptr(ws), ws.numel(), _ptr(status), cs))
    else:
        tm = out.get("true_mask") if true_mask else None
        _check(lib.sparse_pattern_capture_ex(_ptr(maps), n, L, lam, tau, mu, eps, SCALINGS[scaling],
                                             _ptr(out["diag_ptr"]), _ptr(out["diag_offsets"]),
                                             _ptr(out["vert_ptr"]), _ptr(out["vert_cols"]), _ptr(tm),
                                             _ptr(ws), ws.numel(), _ptr(status), cs))
    if check:
        _check_status(status, s)
    return out


# ------------------------------------------------------------------------------------
# Stage two
# ------------------------------------------------------------------------------------

class Plan:
    """A compiled plan: the extended lists and the tile lists, as CUDA tensors."""

    def __init__(self, sizes: PlanSizes, device):
        self.sizes = sizes
        H, nqb, T = sizes.n_heads, sizes.nqb, max(int(sizes.n_tiles), 1)
        i32 = dict(dtype=torch.int32, device=device)
        self.ext_diag_ptr = torch.empty(H + 1, **i32)
        self.ext_diag_offsets = torch.empty(max(sizes.n_diag, 1), **i32)
        self.ext_vert_ptr = torch.empty(H + 1, **i32)
        self.ext_vert_cols = torch.empty(max(sizes.n_vert, 1), **i32)
        self.tile_ptr = torch.empty(H * nqb + 1, **i32)
        self.tile_key0 = torch.empty(T, **i32)
        self.tile_dmask = torch.empty((T, 4), dtype=torch.int64, device=device)
        self.tile_cmask = torch.empty((T, 2), dtype=torch.int64, device=device)
        self.tile_flags = torch.empty(T, **i32)
        self.stripe_cnt = torch.empty(H * nqb, **i32)
        st = PlanStruct()
        st.n_heads, st.S, st.nqb, st.max_vert = H, sizes.S, nqb, sizes.max_vert
        st.n_tiles = int(sizes.n_tiles)
        st.n_diag, st.n_vert = int(sizes.n_diag), int(sizes.n_vert)
        for name in ("ext_diag_ptr", "ext_diag_offsets", "ext_vert_ptr", "ext_vert_cols", "tile_ptr",
                     "tile_key0", "tile_dmask", "tile_cmask", "tile_flags", "stripe_cnt"):
            setattr(st, name, getattr(self, name).data_ptr())
        self.tile_bits = None
        if sizes.bitmap_slots > 0:  # Case-2 plan: element bitmaps, 128 rows x 2 words per slot
            self.tile_bits = torch.empty((H * sizes.bitmap_slots, 128, 2), dtype=torch.int64, device=device)
            st.bitmap_slots = sizes.bitmap_slots
            st.tile_bits = self.tile_bits.data_ptr()
        self.struct = st

    @property
    def S(self):
        return self.sizes.S

    @property
    def n_heads(self):
        return self.sizes.n_heads

    @property
    def n_tiles(self):
        return int(self.sizes.n_tiles)

    def to_numpy(self):
        """Host copies in the oracle's layout (uint64 masks, uint32 flags)."""
        T = self.n_tiles
        out = dict(tile_ptr=self.tile_ptr.cpu().numpy(), tile_key0=self.tile_key0[:T].cpu().numpy(),
                   tile_dmask=self.tile_dmask[:T].cpu().numpy().view("uint64"),
                   tile_cmask=self.tile_cmask[:T].cpu().numpy().view("uint64"),
                   tile_flags=self.tile_flags[:T].cpu().numpy().view("uint32"),
                   stripe_cnt=self.stripe_cnt.cpu().numpy())
        if self.tile_bits is not None:
            out["tile_bits"] = self.tile_bits.cpu().numpy().view("uint64")
        edp = self.ext_diag_ptr.cpu().numpy()
        evp = self.ext_vert_ptr.cpu().numpy()
        out["ext"] = (edp, self.ext_diag_offsets.cpu().numpy()[:edp[-1]], evp,
                      self.ext_vert_cols.cpu().numpy()[:evp[-1]])
        return out


def extend(diag_ptr, diag_offsets, vert_ptr, vert_cols, S: int, *, stream=None, check: bool = True,
           ws=None, status=None, sizes_only: bool = False, true_mask=None):
    """sparse_pattern_extend: sizing pass (synchronises) then fill pass.  Returns a Plan.
    With true_mask (the capture's bitmap, int32 [H, L, ceil(L/32)] on the device) it is
    sparse_pattern_extend_case2: the first L x L block keeps the true mask."""
    lib = load()
    for t, nm in ((diag_ptr, "diag_ptr"), (diag_offsets, "diag_offsets"), (vert_ptr, "vert_ptr"),
                  (vert_cols, "vert_cols")):
        _need_cuda(t, nm, torch.int32)
    H = diag_ptr.numel() - 1
    if vert_ptr.numel() != H + 1:
        raise SSAError(-1, "diag_ptr and vert_ptr must describe the same number of heads")
    dev = diag_ptr.device
    # an empty value list is a zero-size tensor without storage; the C ABI wants a
    # valid pointer even when no entry is read
    if diag_offsets.numel() == 0:
        diag_offsets = torch.zeros(1, dtype=torch.int32, device=dev)
    if vert_cols.numel() == 0:
        vert_cols = torch.zeros(1, dtype=torch.int32, device=dev)
    need = lib.sparse_pattern_extend_ws_bytes(H, S)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    cs, s = _stream(stream)
    sizes = PlanSizes()
    if true_mask is not None:
        L = _check_true_mask(true_mask, H)
        run = lambda pl: lib.sparse_pattern_extend_case2(H, _ptr(diag_ptr), _ptr(diag_offsets), _ptr(vert_ptr),
                                                         _ptr(vert_cols), _ptr(true_mask), L, S, C.byref(sizes),
                                                         pl, _ptr(ws), ws.numel(), _ptr(status), cs)
    else:
        run = lambda pl: lib.sparse_pattern_extend(H, _ptr(diag_ptr), _ptr(diag_offsets), _ptr(vert_ptr),
                                                   _ptr(vert_cols), S, C.byref(sizes), pl, _ptr(ws), ws.numel(),
                                                   _ptr(status), cs)
    _check(run(None))
    if sizes_only:
        return sizes
    plan = Plan(sizes, dev)
    plan._ws = ws
    plan._true_mask = true_mask
    _check(run(C.byref(plan.struct)))
    if check:
        _check_status(status, s)
    return plan


def _check_true_mask(true_mask, H):
    _need_cuda(true_mask, "true_mask", torch.int32)
    if true_mask.dim() != 3 or true_mask.shape[0] != H or true_mask.shape[2] != (true_mask.shape[1] + 31) // 32:
        raise SSAError(-1, "true_mask must be [H, L, ceil(L/32)] int32")
    return true_mask.shape[1]


def refill(plan: Plan, diag_ptr, diag_offsets, vert_ptr, vert_cols, *, true_mask=None, stream=None,
           status=None):
    """Re-run only the fill pass of sparse_pattern_extend into an existing plan (same sizes).
    A Case-2 plan (made with a true mask) is refilled through sparse_pattern_extend_case2
    with `true_mask` (by default the mask it was made with).  Nothing synchronises: a new
    plan that does not fit leaves the plan as it was and sets SSA_ERR_CAPACITY in status."""
    lib = load()
    for t, nm in ((diag_ptr, "diag_ptr"), (diag_offsets, "diag_offsets"), (vert_ptr, "vert_ptr"),
                  (vert_cols, "vert_cols")):
        _need_cuda(t, nm, torch.int32)
    H, S = plan.n_heads, plan.S
    if diag_ptr.numel() != H + 1 or vert_ptr.numel() != H + 1:
        raise SSAError(-1, f"diag_ptr and vert_ptr must hold {H + 1} offsets (the plan's heads + 1)")
    if diag_offsets.numel() == 0:
        diag_offsets = torch.zeros(1, dtype=torch.int32, device=diag_ptr.device)
    if vert_cols.numel() == 0:
        vert_cols = torch.zeros(1, dtype=torch.int32, device=diag_ptr.device)
    if status is not None:
        _need_cuda(status, "status", torch.int32)
    cs, _ = _stream(stream)
    lists = (_ptr(diag_ptr), _ptr(diag_offsets), _ptr(vert_ptr), _ptr(vert_cols))
    if plan.tile_bits is not None:
        tm = getattr(plan, "_true_mask", None) if true_mask is None else true_mask
        if tm is None:
            raise SSAError(-1, "refilling a Case-2 plan needs its true_mask")
        L = _check_true_mask(tm, H)
        _check(lib.sparse_pattern_extend_case2(H, *lists, _ptr(tm), L, S, C.byref(plan.sizes),
                                               C.byref(plan.struct), _ptr(plan._ws), plan._ws.numel(),
                                               _ptr(status), cs))
        plan._true_mask = tm
    else:
        if true_mask is not None:
            raise SSAError(-1, "a plan made without a true mask has no bitmap tiles: "
                               "make it with extend(..., true_mask=...)")
        _check(lib.sparse_pattern_extend(H, *lists, S, C.byref(plan.sizes), C.byref(plan.struct),
                                         _ptr(plan._ws), plan._ws.numel(), _ptr(status), cs))


# ------------------------------------------------------------------------------------
# Attention
# ------------------------------------------------------------------------------------

def attn_ws_bytes(plan: Plan, d: int) -> int:
    return int(load().sparse_attn_fwd_ws_bytes(plan.n_heads, plan.sizes.max_vert, d))


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan: Plan, *, kv_map=None,
             scale: float | None = None, out=None, lse=None, ws=None, stream=None, check: bool = True,
             status=None):
    """sparse_attn_fwd.  q [H_q,S,d], k/v [H_kv,S,d] bf16 CUDA.  Returns (O bf16, LSE fp32)."""
    lib = load()
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _need_cuda(t, nm, torch.bfloat16)
    Hq, S, d = q.shape
    Hkv = k.shape[0]
    if k.shape != (Hkv, S, d) or v.shape != (Hkv, S, d):
        raise SSAError(-1, "k and v must be [H_kv, S, d] matching q")
    dev = q.device
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, S), dtype=torch.float32, device=dev)
    need = lib.sparse_attn_fwd_ws_bytes(Hq, plan.sizes.max_vert, d)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if kv_map is not None:
        _need_cuda(kv_map, "kv_map", torch.int32)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    cs, s = _stream(stream)
    _check(lib.sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, S, d, C.byref(plan.struct),
                               _ptr(kv_map), float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                               _ptr(status), cs))
    if check:
        _check_status(status, s)
    return out, lse


# ------------------------------------------------------------------------------------
# Decoding step
# ------------------------------------------------------------------------------------

def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, pos: torch.Tensor,
                plan: Plan, *, kv_map=None, scale: float | None = None, out=None, lse=None, ws=None,
                stream=None, check: bool = True, status=None):
    """sparse_attn_decode.  q [B,H_q,d], caches [B,H_kv,S,d] bf16, pos [B] int32 (CUDA).
    Returns (O [B,H_q,d] bf16, LSE [B,H_q] fp32)."""
    lib = load()
    for t, nm in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_cuda(t, nm, torch.bfloat16)
    _need_cuda(pos, "pos", torch.int32)
    B, Hq, d = q.shape
    Hkv, S = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, S, d) or v_cache.shape != k_cache.shape:
        raise SSAError(-1, "k_cache and v_cache must be [B, H_kv, S, d] matching q")
    if pos.numel() != B:
        raise SSAError(-1, "pos must hold one position per sequence")
    dev = q.device
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    need = lib.sparse_attn_decode_ws_bytes(B, Hq, d)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if kv_map is not None:
        _need_cuda(kv_map, "kv_map", torch.int32)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    cs, s = _stream(stream)
    _check(lib.sparse_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), B, Hq, Hkv, S, d, _ptr(pos),
                                  C.byref(plan.struct), _ptr(kv_map), float(scale), _ptr(out), _ptr(lse),
                                  _ptr(ws), ws.numel(), _ptr(status), cs))
    if check:
        _check_status(status, s)
    return out, lse
