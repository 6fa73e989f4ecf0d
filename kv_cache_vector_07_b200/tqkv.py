"""Python binding of libtqkv: argument marshalling only.

Every function mirrors one C entry point of ``include/tqkv.h`` and passes
torch tensors as raw device pointers plus the current CUDA stream.  All
computation happens in the library's CUDA kernels; there is no fallback: if
``libtqkv.so`` is missing or fails to load, importing this module raises.
Workspaces are allocated here with torch (zero-filled) when the caller does
not pass one; the library itself never allocates device memory outside
``tq_make_params``.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtqkv.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "tqkv.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtqkv.so is not built ({LIB_PATH}); run `python -m kv_cache_vector_07_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ECUDA, TQ_EDEVICE, TQ_ENOMEM, TQ_ESCRATCH = range(7)
TQ_NOALLOC_SCRATCH_BYTES = 16 << 20
TQ_DEV_SLOT_RANGE, TQ_DEV_BLOCK_RANGE, TQ_DEV_WAIT_TIMEOUT = 0x1, 0x2, 0x4
TQ_DTYPE_BF16, TQ_DTYPE_F32 = 0, 1
TQ_ROT_HADAMARD, TQ_ROT_DENSE = 0, 1
TQ_BITS_HALF = 16
TQ_BITS_POLAR = 32


def half_bits(rate: float) -> int:
    """Code width of a fractional rate (1.5, 2.5, 3.5): TQ_BITS_HALF | b."""
    b = int(rate - 0.5)
    if rate - 0.5 != b or not 1 <= b <= 3:
        raise ValueError("fractional rates are 1.5, 2.5 and 3.5")
    return TQ_BITS_HALF | b


def _n_levels(bits: int, d: int) -> tuple[int, int]:
    if bits == 8:
        return 0, 0
    if bits == TQ_BITS_POLAR:
        lv = int(np.log2(d))
        return 16 + 4 * (lv - 1), 15 + 3 * (lv - 1)
    if bits & TQ_BITS_HALF:
        b = bits & 7
        return (2 << b) + (1 << b), (2 << b) + (1 << b) - 2
    return 1 << bits, (1 << bits) - 1

_vp, _i32, _i64, _u64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t


class CacheDesc(ctypes.Structure):
    """Mirror of tq_cache_desc."""
    _fields_ = [("d", _i32), ("kbits", _i32), ("kqjl", _i32), ("vbits", _i32), ("page_tokens", _i32),
                ("n_kv_heads", _i32)]

    def __repr__(self):
        return (f"CacheDesc(d={self.d}, kbits={self.kbits}, kqjl={self.kqjl}, vbits={self.vbits}, "
                f"page_tokens={self.page_tokens}, n_kv_heads={self.n_kv_heads})")


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("tq_make_params", _i32, [_i32, _i32, _u64, ctypes.POINTER(_vp)])
_sig("tq_make_params_rot", _i32, [_i32, _i32, _u64, _i32, ctypes.POINTER(_vp)])
_sig("tq_compute_rotation_host", _i32, [_i32, _u64, _i32, _vp])
_sig("tq_params_export_rotation", _i32, [_vp, _vp])
_sig("tq_compute_params_host", _i32, [_i32, _i32, _u64, _vp, _vp, _vp, _vp])
_sig("tq_free_params", None, [_vp])
_sig("tq_params_export", _i32, [_vp, _vp, _vp, _vp, _vp])
_sig("tq_cache_bytes", _i32, [ctypes.POINTER(CacheDesc), ctypes.POINTER(_sz)])
_sig("tq_encode_workspace_bytes", _sz, [ctypes.POINTER(CacheDesc), _i64])
_sig("tq_encode", _i32, [_vp, _vp, ctypes.POINTER(CacheDesc), _vp, _vp, _i32, _i64, _vp, _vp, _i64, _vp, _sz,
                         _vp])
_sig("tq_decode_workspace_bytes", _sz, [ctypes.POINTER(CacheDesc), _i32, _i32, _i32])
_sig("tq_decode_attn", _i32, [_vp, _vp, ctypes.POINTER(CacheDesc), _vp, _i32, _i32, _vp, _i32, _vp, _i32, _vp,
                              _i64, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("tq_decode_attn_noalloc", _i32, [_vp, _vp, ctypes.POINTER(CacheDesc), _vp, _i32, _i32, _vp, _i32, _vp, _i32,
                                      _vp, _i64, _vp, _vp, _vp, _i64, _vp])
_sig("tq_decode_step", _i32, [_vp, _vp, ctypes.POINTER(CacheDesc), _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32, _vp,
                              _i32, _vp, _i64, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("tq_prefill_workspace_bytes", _sz, [ctypes.POINTER(CacheDesc), _i32, _i32, _i32])
_sig("tq_prefill_attn", _i32, [_vp, _vp, ctypes.POINTER(CacheDesc), _vp, _i32, _i32, _vp, _i32, _i32, _vp, _i64,
                               _vp, _vp, _vp, _sz, _vp])
_sig("tq_score_workspace_bytes", _sz, [ctypes.POINTER(CacheDesc), _i64, _i32, _i32])
_sig("tq_score", _i32, [_vp, ctypes.POINTER(CacheDesc), _vp, _i64, _vp, _i32, _i32, _vp, _vp, _vp, _sz, _vp])
_sig("tq_read_status", _i32, [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)])
_sig("tq_status_string", ctypes.c_char_p, [_i32])
_sig("tq_test_stall_next_decode", _i32, [ctypes.c_uint32])
_sig("tq_noalloc_read_status", _i32, [_vp, ctypes.POINTER(ctypes.c_uint32)])


class TQError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return _lib.tq_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != TQ_OK:
        raise TQError(code, where)


def declared_functions() -> list[str]:
    """Names of the functions declared in include/tqkv.h."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def exported(name: str) -> bool:
    try:
        getattr(_lib, name)
        return True
    except AttributeError:
        return False


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev_check(*tensors):
    for t in tensors:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libtqkv arguments must be contiguous CUDA tensors")


# ---------------------------------------------------------------------------
# parameters
# ---------------------------------------------------------------------------
class Params:
    """Handle of library-owned parameters (tq_make_params)."""

    def __init__(self, d: int, bits: int, seed: int, rotation: int = TQ_ROT_HADAMARD):
        h = _vp()
        _check(_lib.tq_make_params_rot(d, bits, seed, rotation, ctypes.byref(h)), "tq_make_params_rot")
        self._h = h
        self.d, self.bits, self.seed, self.rotation = d, bits, seed, rotation

    def rotation_matrix(self) -> np.ndarray:
        """tq_params_export_rotation: R [d, d] (y = R x), float32."""
        R = np.zeros((self.d, self.d), np.float32)
        _check(_lib.tq_params_export_rotation(self._h, R.ctypes.data), "tq_params_export_rotation")
        return R

    @property
    def handle(self):
        return self._h

    def export(self):
        d = self.d
        signs = np.zeros(d, np.int8)
        S = np.zeros((d, d), np.float32)
        L, NB = _n_levels(self.bits, d)
        lv = np.zeros(max(L, 1), np.float32)
        bd = np.zeros(max(NB, 1), np.float32)
        _check(_lib.tq_params_export(self._h, signs.ctypes.data, S.ctypes.data, lv.ctypes.data, bd.ctypes.data),
               "tq_params_export")
        return signs, S, (lv if L else None), (bd if L else None)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.tq_free_params(h)
            self._h = _vp()


def make_params(d: int, bits: int, seed: int, rotation: int = TQ_ROT_HADAMARD) -> Params:
    return Params(d, bits, seed, rotation)


def compute_rotation_host(d: int, seed: int, rotation: int = TQ_ROT_DENSE) -> np.ndarray:
    """tq_compute_rotation_host: the rotation matrix of (d, seed) on the host."""
    R = np.zeros((d, d), np.float32)
    _check(_lib.tq_compute_rotation_host(d, seed, rotation, R.ctypes.data), "tq_compute_rotation_host")
    return R


def compute_params_host(d: int, bits: int, seed: int):
    signs = np.zeros(d, np.int8)
    S = np.zeros((d, d), np.float32)
    L, NB = _n_levels(bits, d)
    lv = np.zeros(max(L, 1), np.float32)
    bd = np.zeros(max(NB, 1), np.float32)
    _check(_lib.tq_compute_params_host(d, bits, seed, signs.ctypes.data, S.ctypes.data, lv.ctypes.data,
                                       bd.ctypes.data), "tq_compute_params_host")
    return signs, S, (lv if L else None), (bd if L else None)


def free_params(p: Params):
    p.__del__()


# ---------------------------------------------------------------------------
# cache
# ---------------------------------------------------------------------------
def cache_desc(d: int, kbits: int, kqjl: bool, vbits: int, page_tokens: int = 64, n_kv_heads: int = 1) -> CacheDesc:
    return CacheDesc(d, kbits, 1 if kqjl else 0, vbits, page_tokens, n_kv_heads)


def cache_bytes(desc: CacheDesc) -> int:
    out = _sz()
    _check(_lib.tq_cache_bytes(ctypes.byref(desc), ctypes.byref(out)), "tq_cache_bytes")
    return int(out.value)


def alloc_cache(desc: CacheDesc, num_blocks: int, device="cuda") -> torch.Tensor:
    """Zeroed cache tensor [num_blocks, n_kv_heads, page_bytes] (uint8)."""
    return torch.zeros((num_blocks, desc.n_kv_heads, cache_bytes(desc)), dtype=torch.uint8, device=device)


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def encode_workspace_bytes(desc: CacheDesc, n_tokens: int) -> int:
    return int(_lib.tq_encode_workspace_bytes(ctypes.byref(desc), n_tokens))


def encode(kp: Params, vp: Params | None, desc: CacheDesc, K: torch.Tensor, V: torch.Tensor | None,
           slot_mapping: torch.Tensor, cache: torch.Tensor, workspace: torch.Tensor | None = None, stream=None):
    """tq_encode: K, V [n_tokens, n_kv_heads, d] (bf16 or fp32) into the cache."""
    _dev_check(K, V, slot_mapping, cache, workspace)
    dt = {torch.bfloat16: TQ_DTYPE_BF16, torch.float32: TQ_DTYPE_F32}.get(K.dtype)
    if dt is None:
        raise ValueError("K must be bf16 or fp32")
    if V is not None and V.dtype != K.dtype:
        raise ValueError("K and V dtypes differ")
    if slot_mapping.dtype != torch.int32:
        raise ValueError("slot_mapping must be int32")
    n_tokens = K.shape[0]
    if workspace is None:
        workspace = _workspace(encode_workspace_bytes(desc, n_tokens), K.device)
    num_blocks = cache.shape[0]
    _check(_lib.tq_encode(kp.handle, vp.handle if vp is not None else None, ctypes.byref(desc), _ptr(K), _ptr(V),
                          dt, n_tokens, _ptr(slot_mapping), _ptr(cache), num_blocks, _ptr(workspace),
                          workspace.numel(), _stream(stream)), "tq_encode")
    return workspace


def decode_workspace_bytes(desc: CacheDesc, B: int, Hq: int, max_seq_len: int) -> int:
    return int(_lib.tq_decode_workspace_bytes(ctypes.byref(desc), B, Hq, max_seq_len))


def decode_attn(kp: Params, vp: Params, desc: CacheDesc, Q: torch.Tensor, block_table: torch.Tensor,
                seq_lens: torch.Tensor, max_seq_len: int, cache: torch.Tensor, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, logits: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None):
    """tq_decode_attn: Q bf16 [B, Hq, d] -> out bf16 [B, Hq, d]."""
    _dev_check(Q, block_table, seq_lens, cache, out, lse, logits, workspace)
    B, Hq, d = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        workspace = _workspace(decode_workspace_bytes(desc, B, Hq, max_seq_len), Q.device)
    stride = logits.shape[-1] if logits is not None else 0
    _check(_lib.tq_decode_attn(kp.handle, vp.handle, ctypes.byref(desc), _ptr(Q), B, Hq, _ptr(block_table),
                               block_table.shape[1], _ptr(seq_lens), max_seq_len, _ptr(cache), cache.shape[0],
                               _ptr(out), _ptr(lse), _ptr(logits), stride, _ptr(workspace), workspace.numel(),
                               _stream(stream)), "tq_decode_attn")
    return out


def decode_step(kp: Params, vp: Params, desc: CacheDesc, K_new: torch.Tensor, V_new: torch.Tensor,
                slot_mapping: torch.Tensor, Q: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor,
                max_seq_len: int, cache: torch.Tensor, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, logits: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None):
    """tq_decode_step: write K_new/V_new bf16 [B, n_kv_heads, d] at slot_mapping
    [B], then decode attention of Q bf16 [B, Hq, d] over seq_lens tokens."""
    _dev_check(K_new, V_new, slot_mapping, Q, block_table, seq_lens, cache, out, lse, logits, workspace)
    if K_new.dtype != torch.bfloat16 or V_new.dtype != torch.bfloat16 or slot_mapping.dtype != torch.int32:
        raise ValueError("K_new/V_new must be bf16 and slot_mapping int32")
    B, Hq, d = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        workspace = _workspace(decode_workspace_bytes(desc, B, Hq, max_seq_len), Q.device)
    stride = logits.shape[-1] if logits is not None else 0
    _check(_lib.tq_decode_step(kp.handle, vp.handle, ctypes.byref(desc), _ptr(K_new), _ptr(V_new),
                               _ptr(slot_mapping), _ptr(Q), B, Hq, _ptr(block_table), block_table.shape[1],
                               _ptr(seq_lens), max_seq_len, _ptr(cache), cache.shape[0], _ptr(out), _ptr(lse),
                               _ptr(logits), stride, _ptr(workspace), workspace.numel(), _stream(stream)),
           "tq_decode_step")
    return out


def decode_attn_noalloc(kp: Params, vp: Params, desc: CacheDesc, Q: torch.Tensor, block_table: torch.Tensor,
                        seq_lens: torch.Tensor, max_seq_len: int, cache: torch.Tensor, out: torch.Tensor | None = None,
                        lse: torch.Tensor | None = None, logits: torch.Tensor | None = None, stream=None):
    """tq_decode_attn_noalloc: tq_decode_attn for callers that cannot allocate
    device memory; the scratch is the library's static device array, shared
    by all calls on the device (calls that overlap on the GPU race)."""
    _dev_check(Q, block_table, seq_lens, cache, out, lse, logits)
    B, Hq, d = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    stride = logits.shape[-1] if logits is not None else 0
    _check(_lib.tq_decode_attn_noalloc(kp.handle, vp.handle, ctypes.byref(desc), _ptr(Q), B, Hq, _ptr(block_table),
                                       block_table.shape[1], _ptr(seq_lens), max_seq_len, _ptr(cache),
                                       cache.shape[0], _ptr(out), _ptr(lse), _ptr(logits), stride, _stream(stream)),
           "tq_decode_attn_noalloc")
    return out


def noalloc_read_status(stream=None) -> int:
    """tq_noalloc_read_status: status flags of the last no-allocation decode
    on the current device (cleared by the read)."""
    flags = ctypes.c_uint32()
    _check(_lib.tq_noalloc_read_status(_stream(stream), ctypes.byref(flags)), "tq_noalloc_read_status")
    return int(flags.value)


def prefill_workspace_bytes(desc: CacheDesc, C: int, Hq: int, seq_len: int) -> int:
    return int(_lib.tq_prefill_workspace_bytes(ctypes.byref(desc), C, Hq, seq_len))


def prefill_attn(kp: Params, vp: Params, desc: CacheDesc, Q: torch.Tensor, block_table: torch.Tensor,
                 seq_len: int, cache: torch.Tensor, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None):
    """tq_prefill_attn: chunk queries Q bf16 [C, Hq, d] over one sequence."""
    _dev_check(Q, block_table, cache, out, lse, workspace)
    C, Hq, d = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        workspace = _workspace(prefill_workspace_bytes(desc, C, Hq, seq_len), Q.device)
    _check(_lib.tq_prefill_attn(kp.handle, vp.handle, ctypes.byref(desc), _ptr(Q), C, Hq, _ptr(block_table),
                                block_table.numel(), seq_len, _ptr(cache), cache.shape[0], _ptr(out), _ptr(lse),
                                _ptr(workspace), workspace.numel(), _stream(stream)), "tq_prefill_attn")
    return out


def score_workspace_bytes(desc: CacheDesc, n_db: int, n_q: int, k: int) -> int:
    return int(_lib.tq_score_workspace_bytes(ctypes.byref(desc), n_db, n_q, k))


def score(p: Params, desc: CacheDesc, db_cache: torch.Tensor, n_db: int, Q: torch.Tensor, k: int,
          top_scores: torch.Tensor | None = None, top_idx: torch.Tensor | None = None,
          workspace: torch.Tensor | None = None, stream=None):
    """tq_score: top-k estimated inner products of fp32 queries Q [n_q, d]."""
    _dev_check(db_cache, Q, top_scores, top_idx, workspace)
    n_q = Q.shape[0]
    if top_scores is None:
        top_scores = torch.empty((n_q, k), dtype=torch.float32, device=Q.device)
    if top_idx is None:
        top_idx = torch.empty((n_q, k), dtype=torch.int64, device=Q.device)
    if workspace is None:
        workspace = _workspace(score_workspace_bytes(desc, n_db, n_q, k), Q.device)
    _check(_lib.tq_score(p.handle, ctypes.byref(desc), _ptr(db_cache), n_db, _ptr(Q), n_q, k, _ptr(top_scores),
                         _ptr(top_idx), _ptr(workspace), workspace.numel(), _stream(stream)), "tq_score")
    return top_scores, top_idx


def read_status(workspace: torch.Tensor, stream=None) -> int:
    flags = ctypes.c_uint32()
    _check(_lib.tq_read_status(_ptr(workspace), _stream(stream), ctypes.byref(flags)), "tq_read_status")
    return int(flags.value)


def test_stall_next_decode(polls: int) -> None:
    """tq_test_stall_next_decode: the next tensor-core decode launch waits
    `polls` polls on a barrier nothing completes and takes its time-out path
    (a testing aid for the TQ_DEV_WAIT_TIMEOUT flag; 0 cancels)."""
    _check(_lib.tq_test_stall_next_decode(int(polls)), "tq_test_stall_next_decode")
