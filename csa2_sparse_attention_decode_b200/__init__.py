"""Python binding of libcsa2 (the CSA2 sparse-attention decode step on B200).

Argument marshalling only: every call forwards torch tensors' device pointers
to the C ABI declared in ``include/csa2.h`` and raises on a non-OK status.
Importing this package loads ``libcsa2.so`` from this directory, building it
with nvcc first when it is missing or older than its sources, and fails
loudly when it can be neither built nor found; there is no other code path.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

LATENT, CODE_BYTES, SCALE_BYTES, KEY_DIM, IDX_HEADS = 512, 256, 32, 128, 32
BLOCK, MAX_BLOCKS, POOL, TOPK, SWA = 8, 2048, 16384, 512, 128
PAGE_ENTRIES, PAGE_BYTES, SWA_BYTES, PENDING_STRIDE = 64, 27648, 66048, 656
PAGE_CODES_BYTES, PAGE_SCALES_BYTES, PAGE_KEYS_BYTES, PAGE_SUMM_BYTES = 16384, 2048, 8192, 1024


def plane_offsets(n_pages: int):
    """Byte offsets of the codes / scales / keys / summaries planes of a pool."""
    return 0, n_pages * 16384, n_pages * 18432, n_pages * 26624
SWA_CODES_OFF, SWA_SCALE_OFF = 0, 65536
INDEX_FLAT, INDEX_FULL, INDEX_REINDEX = 0, 1, 2

EXPORTS = ("csa2_page_bytes", "csa2_swa_bytes", "csa2_workspace_bytes", "csa2_prefill", "csa2_append",
           "csa2_index", "csa2_attend", "csa2_get_device_error", "csa2_status_string", "csa2_set_profile_events",
           "csa2_launch_count", "csa2_attend_noalloc", "csa2_topk", "csa2_shard_blocks", "csa2_shard_pool",
           "csa2_shard_rescore", "csa2_shard_topk", "csa2_attend_partial", "csa2_combine",
           "csa2_selftest_wait_timeout")
MAX_SHARDS = 8
ATTEND_NOALLOC_MAX_ROWS = 512
KERNEL_BLOCK_SCORE, KERNEL_FLAT_SCORE, KERNEL_POOL_SCORE, KERNEL_SELECT, KERNEL_ATTEND, KERNEL_COMBINE = range(6)


class CSA2Error(RuntimeError):
    def __init__(self, call: str, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{call} failed: {status_string(status)} ({status}){detail}")


class csa2_cache(C.Structure):
    _fields_ = [("pool", C.c_void_p), ("n_pages", C.c_int32), ("page_table", C.c_void_p),
                ("max_pages", C.c_int32), ("n_tokens", C.c_void_p), ("m", C.c_void_p), ("swa", C.c_void_p),
                ("pending", C.c_void_p), ("error", C.c_void_p), ("batch", C.c_int32)]


def _load():
    from . import build as _build
    if not _build.up_to_date():
        try:
            _build.build()
        except (OSError, subprocess.CalledProcessError) as e:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libcsa2.so is not built at {LIB_PATH} and building it failed: {e}") from e
    L = C.CDLL(LIB_PATH)
    P, I32, SZ = C.c_void_p, C.c_int32, C.c_size_t
    sig = {
        "csa2_page_bytes": (SZ, []),
        "csa2_swa_bytes": (SZ, []),
        "csa2_workspace_bytes": (SZ, [I32, I32]),
        "csa2_prefill": (C.c_int, [P, I32, I32, I32, I32, I32, P, P, P, P]),
        "csa2_append": (C.c_int, [P, P, P, P, P, P]),
        "csa2_index": (C.c_int, [P, C.c_int, P, P, P, P, P, P, SZ, P]),
        "csa2_attend": (C.c_int, [P, I32, P, P, C.c_float, P, I32, C.c_uint32, P, SZ, P]),
        "csa2_get_device_error": (C.c_int, [P, C.POINTER(C.c_int32), P]),
        "csa2_status_string": (C.c_char_p, [C.c_int]),
        "csa2_set_profile_events": (C.c_int, [I32, P, P]),
        "csa2_attend_noalloc": (C.c_int, [P, I32, P, P, C.c_float, P, I32, P]),
        "csa2_launch_count": (C.c_uint64, []),
        "csa2_topk": (C.c_int, [P, C.c_int64, P, I32, I32, P, P]),
        "csa2_shard_blocks": (C.c_int, [P, P, P, P, P, P, P, SZ, P]),
        "csa2_shard_pool": (C.c_int, [P, P, I32, P, P, P, P, P]),
        "csa2_shard_rescore": (C.c_int, [P, P, P, P, P, P, P, P, P]),
        "csa2_shard_topk": (C.c_int, [P, P, I32, P, P, P, P]),
        "csa2_attend_partial": (C.c_int, [P, I32, P, P, C.c_float, I32, P, P, C.c_uint32, P]),
        "csa2_combine": (C.c_int, [I32, P, P, I32, I32, P, I32, P]),
        "csa2_selftest_wait_timeout": (C.c_int, [P, C.c_uint32, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.csa2_status_string(status).decode()


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libcsa2 takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libcsa2 takes contiguous tensors")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _check(name, st):
    if st != 0:
        raise CSA2Error(name, st)


class Cache:
    """Device storage of a batch of requests' CSA2 caches (allocated by torch)
    plus the matching C struct."""

    def __init__(self, page_table: torch.Tensor, n_pages: int, m, device="cuda"):
        self.device = torch.device(device)
        self.batch = int(page_table.shape[0])
        self.max_pages = int(page_table.shape[1])
        self.n_pages = int(n_pages)
        self.pool = torch.zeros(self.n_pages * PAGE_BYTES, dtype=torch.uint8, device=self.device)
        self.page_table = page_table.to(self.device, torch.int32).contiguous()
        self.n_tokens = torch.zeros(self.batch, dtype=torch.int32, device=self.device)
        self.m = torch.as_tensor(m, dtype=torch.int32).to(self.device).contiguous()
        self.m_host = [int(x) for x in torch.as_tensor(m)]
        self.swa = torch.zeros(self.batch * SWA_BYTES, dtype=torch.uint8, device=self.device)
        self.pending = torch.zeros(self.batch * PENDING_STRIDE, dtype=torch.float32, device=self.device)
        self.error = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.c = csa2_cache(self.pool.data_ptr(), self.n_pages, self.page_table.data_ptr(), self.max_pages,
                            self.n_tokens.data_ptr(), self.m.data_ptr(), self.swa.data_ptr(),
                            self.pending.data_ptr(), self.error.data_ptr(), self.batch)

    @property
    def ref(self):
        return C.byref(self.c)

    @property
    def max_entries(self) -> int:
        return self.max_pages * PAGE_ENTRIES

    # Views of the packed bytes (for tests and inspection).
    def page_view(self) -> torch.Tensor:
        return self.pool.view(self.n_pages, PAGE_BYTES)

    def swa_view(self) -> torch.Tensor:
        return self.swa.view(self.batch, SWA_BYTES)


def csa2_page_bytes() -> int:
    return int(lib.csa2_page_bytes())


def csa2_swa_bytes() -> int:
    return int(lib.csa2_swa_bytes())


def csa2_workspace_bytes(batch: int, max_entries: int) -> int:
    return int(lib.csa2_workspace_bytes(batch, max_entries))


def workspace(cache: Cache) -> torch.Tensor:
    n = csa2_workspace_bytes(cache.batch, cache.max_entries)
    return torch.empty(n, dtype=torch.uint8, device=cache.device)


def csa2_prefill(cache: Cache, req: int, tok_begin: int, n_tok_final: int, lat, key, gate, stream=None):
    n = int(key.shape[0])
    _check("csa2_prefill", lib.csa2_prefill(cache.ref, req, cache.m_host[req], tok_begin, n, n_tok_final,
                                            _ptr(lat), _ptr(key), _ptr(gate), _stream(stream)))


def csa2_append(cache: Cache, lat, key, gate, n_new, stream=None):
    _check("csa2_append", lib.csa2_append(cache.ref, _ptr(lat), _ptr(key), _ptr(gate), _ptr(n_new),
                                          _stream(stream)))


def csa2_index(cache: Cache, mode: int, q_idx, w, pool, pool_len, topk, ws, stream=None):
    qi = q_idx.view(torch.int16) if q_idx.dtype == torch.bfloat16 else q_idx
    _check("csa2_index", lib.csa2_index(cache.ref, mode, _ptr(qi), _ptr(w), _ptr(pool), _ptr(pool_len),
                                        _ptr(topk), _ptr(ws), ws.numel(), _stream(stream)))


def csa2_topk(scores, n, k: int, out, stream=None):
    """Top-k of each row of scores [batch, stride] (f32), first n[b] elements
    (n int32 [batch]); out int32 [batch, k] gets ascending indices, -1 padded."""
    assert scores.dtype == torch.float32 and scores.stride(1) == 1 and n.dtype == torch.int32
    assert out.dtype == torch.int32 and out.is_contiguous() and tuple(out.shape) == (scores.shape[0], k)
    _check("csa2_topk", lib.csa2_topk(_ptr(scores), scores.stride(0), _ptr(n), int(scores.shape[0]), int(k),
                                      _ptr(out), _stream(stream)))


ATTEND_INPUTS_SETTLED = 1


def csa2_attend(cache: Cache, q, topk, scale: float, out, ws, stream=None, flags: int = 0):
    heads = int(q.shape[1])
    qq = q.view(torch.int16) if q.dtype == torch.bfloat16 else q
    fp32 = 1 if out.dtype == torch.float32 else 0
    _check("csa2_attend", lib.csa2_attend(cache.ref, heads, _ptr(qq), _ptr(topk), float(scale), _ptr(out), fp32,
                                          flags, _ptr(ws), ws.numel(), _stream(stream)))


def csa2_get_device_error(cache: Cache, stream=None) -> int:
    code = C.c_int32(0)
    st = lib.csa2_get_device_error(cache.ref, C.byref(code), _stream(stream))
    if st not in (0, 4):
        raise CSA2Error("csa2_get_device_error", st)
    return int(code.value)


def csa2_set_profile_events(kernel: int, start=None, stop=None):
    """Bracket every later launch of `kernel` with torch.cuda.Event pair
    (start, stop) recorded on the launching stream; None/None turns it off."""
    a = C.c_void_p(start.cuda_event) if start is not None else None
    b = C.c_void_p(stop.cuda_event) if stop is not None else None
    _check("csa2_set_profile_events", lib.csa2_set_profile_events(kernel, a, b))


def csa2_launch_count() -> int:
    return int(lib.csa2_launch_count())


def csa2_attend_noalloc(cache: Cache, q, topk, scale: float, out, stream=None) -> int:
    """csa2_attend without a workspace, for callers that cannot allocate
    device memory: the library keeps the split partials in its own fixed
    array (batch * heads <= ATTEND_NOALLOC_MAX_ROWS).  Returns the C status;
    raises on anything but OK or CSA2_ERR_UNSUPPORTED (size over the limit)."""
    heads = int(q.shape[1])
    qq = q.view(torch.int16) if q.dtype == torch.bfloat16 else q
    fp32 = 1 if out.dtype == torch.float32 else 0
    st = lib.csa2_attend_noalloc(cache.ref, heads, _ptr(qq), _ptr(topk), float(scale), _ptr(out), fp32,
                                 _stream(stream))
    if st not in (0, 2):
        raise CSA2Error("csa2_attend_noalloc", st)
    return int(st)


# ---------------------------------------------------------------- sequence shards
def _ptrs(ts):
    """Host array of the device pointers of tensors ts (kept alive by the caller)."""
    if not 1 <= len(ts) <= MAX_SHARDS:
        raise ValueError(f"1..{MAX_SHARDS} shards, got {len(ts)}")
    arr = (C.c_void_p * len(ts))(*[_ptr(t).value for t in ts])
    return C.cast(arr, C.c_void_p), arr


def _bits16(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def csa2_shard_blocks(cache, entry_offset, q_idx, w, block_ids, block_scores, ws, stream=None):
    _check("csa2_shard_blocks", lib.csa2_shard_blocks(cache.ref, _ptr(entry_offset), _ptr(_bits16(q_idx)), _ptr(w),
                                                      _ptr(block_ids), _ptr(block_scores), _ptr(ws), ws.numel(),
                                                      _stream(stream)))


def csa2_shard_pool(cache, entry_offset, cand_ids, cand_scores, pool, pool_len, stream=None):
    pi, ki = _ptrs(cand_ids)
    ps, ks = _ptrs(cand_scores)
    _check("csa2_shard_pool", lib.csa2_shard_pool(cache.ref, _ptr(entry_offset), len(cand_ids), pi, ps, _ptr(pool),
                                                  _ptr(pool_len), _stream(stream)))
    del ki, ks


def csa2_shard_rescore(cache, entry_offset, q_idx, w, pool, pool_len, ids, scores, stream=None):
    _check("csa2_shard_rescore", lib.csa2_shard_rescore(cache.ref, _ptr(entry_offset), _ptr(_bits16(q_idx)), _ptr(w),
                                                        _ptr(pool), _ptr(pool_len), _ptr(ids), _ptr(scores),
                                                        _stream(stream)))


def csa2_shard_topk(cache, entry_offset, cand_ids, cand_scores, topk, stream=None):
    pi, ki = _ptrs(cand_ids)
    ps, ks = _ptrs(cand_scores)
    _check("csa2_shard_topk", lib.csa2_shard_topk(cache.ref, _ptr(entry_offset), len(cand_ids), pi, ps, _ptr(topk),
                                                  _stream(stream)))
    del ki, ks


def csa2_attend_partial(cache, q, topk, scale: float, with_window: bool, o, lse, stream=None, flags: int = 0):
    assert o.dtype == torch.float32 and lse.dtype == torch.float32
    _check("csa2_attend_partial", lib.csa2_attend_partial(cache.ref, int(q.shape[1]), _ptr(_bits16(q)), _ptr(topk),
                                                          float(scale), 1 if with_window else 0, _ptr(o), _ptr(lse),
                                                          flags, _stream(stream)))


def csa2_combine(o_parts, lse_parts, out, stream=None):
    """out [batch, heads, 512] (bf16 or f32) = log-sum-exp merge of the
    partial results o_parts[s] [batch, heads, 512] f32 with lse_parts[s]
    [batch, heads] f32."""
    if len(o_parts) != len(lse_parts):
        raise ValueError("one lse per partial output")
    po, ko = _ptrs(o_parts)
    pl, kl = _ptrs(lse_parts)
    fp32 = 1 if out.dtype == torch.float32 else 0
    _check("csa2_combine", lib.csa2_combine(len(o_parts), po, pl, int(out.shape[0]), int(out.shape[1]), _ptr(out),
                                            fp32, _stream(stream)))
    del ko, kl


def csa2_selftest_wait_timeout(error_word, polls: int = 1024, stream=None):
    """Run the bounded-wait self-test: error_word (int32 device tensor of one
    element) receives CSA2_DEV_TIMEOUT once the probe's wait runs out."""
    _check("csa2_selftest_wait_timeout", lib.csa2_selftest_wait_timeout(_ptr(error_word), int(polls), _stream(stream)))
