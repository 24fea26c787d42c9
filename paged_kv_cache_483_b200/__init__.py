"""Python binding of libpagedattn.so (B200 paged attention).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels; PyTorch supplies device memory and streams.  There is no CPU or
PyTorch fallback -- if the shared library is missing this module raises.

The raw C ABI is exposed under the same names as ``include/pa.h``
(``pa_pool_create``, ``pa_append_kv``, ``pa_cow_copy``, ``pa_decode``,
``pa_prefill_chunk``, ``pa_free`` ...) via :func:`lib`; :class:`Pool` is a
small convenience layer that keeps the borrowed cache tensors alive.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_F32, PA_BF16, PA_INT8, PA_FP8 = 0, 1, 2, 3
PA_INT8_RECORD_BYTES = 4224   # one (block, head) record of an int8 or FP8 pool
STATUS = {0: "ok", 1: "invalid argument", 2: "unknown sequence", 3: "duplicate sequence",
          4: "pool exhausted", 5: "CUDA error", 6: "device error", 7: "unsupported",
          8: "host-only pool", 9: "broken invariant", 10: "scratch limit"}
PA_DEVERR_BLOCK_ID, PA_DEVERR_SLOT, PA_DEVERR_KV_LEN, PA_DEVERR_TIMEOUT = 1, 2, 4, 8

EXPORTS = ["pa_pool_create", "pa_free", "pa_seq_create", "pa_seq_fork", "pa_seq_release",
           "pa_seq_table", "pa_block_tables", "pa_plan_append", "pa_pool_stats",
           "pa_refcounts", "pa_validate", "pa_append_kv", "pa_reshape_and_cache",
           "pa_cow_copy", "pa_decode_workspace_bytes", "pa_decode", "pa_prefill_chunk",
           "pa_get_error", "pa_status_string", "pa_decode_path", "pa_prefill_path",
           "pa_decode_static_scratch", "pa_decode_append", "pa_seq_create_cached",
           "pa_prefix_publish", "pa_prefix_clear", "pa_prefix_entries", "pa_pool_create_int8",
           "pa_decode_window", "pa_decode_window_workspace_bytes", "pa_pool_create_layers",
           "pa_pool_layer", "pa_decode_window_append", "pa_pool_create_fp8", "pa_seq_truncate",
           "pa_batch_create", "pa_batch_step", "pa_batch_rollback", "pa_batch_set_window",
           "pa_batch_sync",
           "pa_batch_free"]


class PAError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({code})")


class Stats(C.Structure):
    _fields_ = [(n, C.c_int64) for n in (
        "allocated_blocks", "free_blocks", "physical_capacity_tokens",
        "physical_payload_tokens", "logical_tokens", "internal_waste_tokens",
        "sharing_savings_tokens", "live_sequences")]


_lib = None
_P, _I32, _I64, _SZ, _F = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t, C.c_float
_PI32, _PI64 = C.POINTER(C.c_int32), C.POINTER(C.c_int64)


def lib():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m paged_kv_cache_483_b200.build`")
    L = C.CDLL(LIB_PATH)
    sig = {
        "pa_pool_create": ([_I32, _I32, _I32, _I32, C.c_int, _P, _P, _PI32, C.POINTER(_P)], C.c_int),
        "pa_free": ([_P], C.c_int),
        "pa_pool_create_layers": ([_I32, _I32, _I32, _I32, C.c_int, _I32, _P, _P, _PI32,
                                   C.POINTER(_P)], C.c_int),
        "pa_pool_layer": ([_P, _I32, C.POINTER(_P)], C.c_int),
        "pa_pool_create_int8": ([_I32, _I32, _I32, _I32, _P, _PI32, C.POINTER(_P)], C.c_int),
        "pa_pool_create_fp8": ([_I32, _I32, _I32, _I32, _P, _PI32, C.POINTER(_P)], C.c_int),
        "pa_seq_create": ([_P, _I32], C.c_int),
        "pa_seq_fork": ([_P, _I32, _I32, _I32], C.c_int),
        "pa_seq_release": ([_P, _I32], C.c_int),
        "pa_seq_truncate": ([_P, _PI32, _PI32, _I32], C.c_int),
        "pa_seq_table": ([_P, _I32, _PI32, _I32, _PI32, _PI32], C.c_int),
        "pa_seq_create_cached": ([_P, _I32, C.c_uint64, C.c_uint64, _PI32, _I32, _PI32], C.c_int),
        "pa_prefix_publish": ([_P, _I32, C.c_uint64, C.c_uint64, _PI32, _I32, _PI32], C.c_int),
        "pa_prefix_clear": ([_P, _PI32], C.c_int),
        "pa_prefix_entries": ([_P], _I64),
        "pa_block_tables": ([_P, _PI32, _I32, _I32, _PI32, _PI32], C.c_int),
        "pa_plan_append": ([_P, _PI32, _PI32, _I32, _PI64, _PI32, _PI32, _I32, _PI32], C.c_int),
        "pa_pool_stats": ([_P, C.POINTER(Stats)], C.c_int),
        "pa_refcounts": ([_P, _PI32], C.c_int),
        "pa_validate": ([_P], C.c_int),
        "pa_append_kv": ([_P, _PI32, _PI32, _I32, _P, _P, _PI64, _P], C.c_int),
        "pa_reshape_and_cache": ([_P, _P, _P, _P, _I32, _P], C.c_int),
        "pa_cow_copy": ([_P, _P, _P, _I32, _P], C.c_int),
        "pa_decode_workspace_bytes": ([_P, _I32, _I32, _I32, _I32], _SZ),
        "pa_decode": ([_P, _P, _I32, _I32, _P, _I32, _P, _F, _I32, _P, _SZ, _P, _P], C.c_int),
        "pa_decode_window": ([_P, _P, _I32, _I32, _P, _I32, _P, _F, _I32, _I32, _I32, _P, _SZ,
                              _P, _P], C.c_int),
        "pa_decode_window_workspace_bytes": ([_P, _I32, _I32, _I32, _I32, _I32, _I32], _SZ),
        "pa_decode_window_append": ([_P, _P, _P, _P, _P, _I32, _I32, _P, _I32, _P, _F, _I32, _I32,
                                     _I32, _P, _SZ, _P, _P], C.c_int),
        "pa_prefill_chunk": ([_P, _P, _I32, _I32, _I32, _P, _I32, _P, _F, _I32, _P, _P],
                             C.c_int),
        "pa_get_error": ([_P, _PI32], C.c_int),
        "pa_status_string": ([C.c_int], C.c_char_p),
        "pa_decode_path": ([_P, _I32], _I32),
        "pa_prefill_path": ([_P, _I32], _I32),
        "pa_decode_static_scratch": ([_P, _P, _I32, _I32, _P, _I32, _P, _F, _I32, _P, _P], C.c_int),
        "pa_decode_append": ([_P, _P, _P, _P, _P, _I32, _I32, _P, _I32, _P, _F, _I32, _P, _SZ, _P,
                              _P], C.c_int),
        "pa_batch_create": ([_P, _PI32, _I32, _I32, _I32, _I32, C.POINTER(_P)], C.c_int),
        "pa_batch_step": ([_P, _P, _P, _P, _F, _P, _P], C.c_int),
        "pa_batch_rollback": ([_P], C.c_int),
        "pa_batch_sync": ([_P], C.c_int),
        "pa_batch_set_window": ([_P, _I32, _I32], C.c_int),
        "pa_batch_free": ([_P], C.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes, f.restype = args, res
    _lib = L
    return L


def _check(code, where):
    if code != 0:
        raise PAError(code, where)


def _i32(arr):
    a = np.ascontiguousarray(arr, dtype=np.int32)
    return a, a.ctypes.data_as(_PI32)


def _stream(stream):
    if stream is None:
        import torch
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _dev_ptr(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (checked)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    return C.c_void_p(t.data_ptr())


class Pool:
    """A physical KV pool [num_blocks, block_size, num_kv_heads, head_dim]
    plus its host block manager.  ``k_cache``/``v_cache`` are borrowed CUDA
    tensors (kept alive here); pass ``None`` for both to get a host-only
    manager (no GPU needed).  ``dtype="int8"`` or ``"fp8"`` (E4M3 codes):
    ``k_cache`` is the uint8 tensor [num_blocks, num_kv_heads,
    PA_INT8_RECORD_BYTES] of packed (block, head) records (layout in
    ``pa.h``) and ``v_cache`` is None; appends and queries are bf16."""

    def __init__(self, num_blocks, block_size, num_kv_heads, head_dim, dtype="bf16",
                 k_cache=None, v_cache=None, alloc_order=None):
        L = lib()
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self.num_kv_heads, self.head_dim = int(num_kv_heads), int(head_dim)
        self.dtype = dtype
        self.k_cache, self.v_cache = k_cache, v_cache
        if dtype in ("int8", "fp8"):
            import torch
            rshape = (self.num_blocks, self.num_kv_heads, PA_INT8_RECORD_BYTES)
            if k_cache is None or tuple(k_cache.shape) != rshape or v_cache is not None:
                raise ValueError(f"an {dtype} pool takes k_cache = uint8 records {rshape} "
                                 "and no v_cache")
            order_arr, order_p = (None, None) if alloc_order is None else _i32(alloc_order)
            h = C.c_void_p()
            fn = "pa_pool_create_int8" if dtype == "int8" else "pa_pool_create_fp8"
            _check(getattr(L, fn)(num_blocks, block_size, num_kv_heads, head_dim,
                                  _dev_ptr(k_cache, torch.uint8, "k_cache"), order_p,
                                  C.byref(h)), fn)
            self._h = h
            self._ws = None
            return
        code = PA_BF16 if dtype == "bf16" else PA_F32
        if k_cache is not None:
            import torch
            want = torch.bfloat16 if dtype == "bf16" else torch.float32
            shape = (self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim)
            for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
                if tuple(t.shape) != shape:
                    raise ValueError(f"{name} must have shape {shape}")
            kp, vp = _dev_ptr(k_cache, want, "k_cache"), _dev_ptr(v_cache, want, "v_cache")
        else:
            kp = vp = None
        order_arr, order_p = (None, None) if alloc_order is None else _i32(alloc_order)
        h = C.c_void_p()
        _check(L.pa_pool_create(num_blocks, block_size, num_kv_heads, head_dim, code,
                                kp, vp, order_p, C.byref(h)), "pa_pool_create")
        self._h = h
        self._ws = None

    @classmethod
    def layered(cls, num_blocks, block_size, num_kv_heads, head_dim, dtype, num_layers,
                k_cache, v_cache=None, alloc_order=None):
        """A pool over caches holding ``num_layers`` layers (leading dimension);
        ``layer(l)`` gives each layer's handle, all sharing one manager."""
        import torch
        self = cls.__new__(cls)
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self.num_kv_heads, self.head_dim = int(num_kv_heads), int(head_dim)
        self.dtype, self.k_cache, self.v_cache = dtype, k_cache, v_cache
        self._ws, self._view = None, False
        code = {"bf16": PA_BF16, "f32": PA_F32, "int8": PA_INT8, "fp8": PA_FP8}[dtype]
        want = {"bf16": torch.bfloat16, "f32": torch.float32, "int8": torch.uint8,
                "fp8": torch.uint8}[dtype]
        order_arr, order_p = (None, None) if alloc_order is None else _i32(alloc_order)
        h = C.c_void_p()
        _check(lib().pa_pool_create_layers(num_blocks, block_size, num_kv_heads, head_dim, code,
                                           num_layers, _dev_ptr(k_cache, want, "k_cache"),
                                           _dev_ptr(v_cache, want, "v_cache"), order_p,
                                           C.byref(h)), "pa_pool_create_layers")
        self._h = h
        self._layers = {0: self}
        return self

    def layer(self, index):
        """Handle of one layer (borrowed: it lives as long as this pool)."""
        if index in getattr(self, "_layers", {}):
            return self._layers[index]
        h = C.c_void_p()
        _check(lib().pa_pool_layer(self._h, int(index), C.byref(h)), "pa_pool_layer")
        v = Pool.__new__(Pool)
        v.__dict__.update({k: val for k, val in self.__dict__.items() if k != "_layers"})
        v._h, v._ws, v._view, v._parent = h, None, True, self
        self._layers[index] = v
        return v

    # -- lifetime ----------------------------------------------------------
    def close(self):
        if getattr(self, "_view", False):
            return                          # a layer handle: freed with its pool
        if getattr(self, "_h", None):
            lib().pa_free(self._h)
            self._h = None
            # the pool's layer handles went with it
            for v in getattr(self, "_layers", {}).values():
                v._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    # -- host block manager -------------------------------------------------
    def create(self, seq):
        _check(lib().pa_seq_create(self._h, int(seq)), "pa_seq_create")

    def fork(self, parent, child, prefix_tokens=-1):
        _check(lib().pa_seq_fork(self._h, int(parent), int(child), int(prefix_tokens)),
               "pa_seq_fork")

    def release(self, seq):
        _check(lib().pa_seq_release(self._h, int(seq)), "pa_seq_release")

    def truncate(self, seqs, lengths):
        """Keep the first lengths[i] tokens of seqs[i] (rollback of the newest
        tokens; all-or-nothing)."""
        seqs_a, sp = _i32(seqs)
        lens_a, lp = _i32(lengths)
        if len(seqs_a) != len(lens_a):
            raise ValueError("seqs and lengths must pair up")
        _check(lib().pa_seq_truncate(self._h, sp, lp, len(seqs_a)), "pa_seq_truncate")

    # -- prefix cache (content-keyed full blocks) ----------------------------
    def create_cached(self, seq, tokens, scope=0, revision=0):
        """New sequence starting with the cached blocks of ``tokens``'s
        longest cached full-block prefix; returns the tokens it covers."""
        toks, tp = _i32(tokens)
        hit = C.c_int32()
        _check(lib().pa_seq_create_cached(self._h, int(seq), int(scope), int(revision), tp,
                                          len(toks), C.byref(hit)), "pa_seq_create_cached")
        return hit.value

    def publish(self, seq, tokens, scope=0, revision=0):
        """Key ``seq``'s full blocks (token ids ``tokens``); returns new keys."""
        toks, tp = _i32(tokens)
        added = C.c_int32()
        _check(lib().pa_prefix_publish(self._h, int(seq), int(scope), int(revision), tp,
                                       len(toks), C.byref(added)), "pa_prefix_publish")
        return added.value

    def prefix_clear(self):
        freed = C.c_int32()
        _check(lib().pa_prefix_clear(self._h, C.byref(freed)), "pa_prefix_clear")
        return freed.value

    def prefix_entries(self):
        return int(lib().pa_prefix_entries(self._h))

    def table(self, seq):
        n, length = C.c_int32(), C.c_int32()
        _check(lib().pa_seq_table(self._h, int(seq), None, 0, C.byref(n), C.byref(length)),
               "pa_seq_table")
        out = np.zeros(max(n.value, 1), np.int32)
        _check(lib().pa_seq_table(self._h, int(seq), out.ctypes.data_as(_PI32), out.size,
                                  C.byref(n), C.byref(length)), "pa_seq_table")
        return out[:n.value].tolist(), length.value

    def block_tables(self, seqs, width):
        seqs_a, sp = _i32(seqs)
        tables = np.zeros((len(seqs_a), width), np.int32)
        lens = np.zeros(len(seqs_a), np.int32)
        _check(lib().pa_block_tables(self._h, sp, len(seqs_a), width,
                                     tables.ctypes.data_as(_PI32), lens.ctypes.data_as(_PI32)),
               "pa_block_tables")
        return tables, lens

    def plan_append(self, seqs, n_new):
        seqs_a, sp = _i32(seqs)
        n_a, np_ = _i32(n_new)
        T = int(np.maximum(n_a, 0).sum())
        slots = np.zeros(max(T, 1), np.int64)
        src = np.zeros(max(len(seqs_a), 1), np.int32)
        dst = np.zeros_like(src)
        ncow = C.c_int32()
        _check(lib().pa_plan_append(self._h, sp, np_, len(seqs_a),
                                    slots.ctypes.data_as(_PI64), src.ctypes.data_as(_PI32),
                                    dst.ctypes.data_as(_PI32), src.size, C.byref(ncow)),
               "pa_plan_append")
        k = ncow.value
        return slots[:T].tolist(), list(zip(src[:k].tolist(), dst[:k].tolist()))

    def stats(self):
        s = Stats()
        _check(lib().pa_pool_stats(self._h, C.byref(s)), "pa_pool_stats")
        return {f: getattr(s, f) for f, _ in Stats._fields_}

    def refcounts(self):
        out = np.zeros(self.num_blocks, np.int32)
        _check(lib().pa_refcounts(self._h, out.ctypes.data_as(_PI32)), "pa_refcounts")
        return out.tolist()

    def validate(self):
        return lib().pa_validate(self._h) == 0

    # -- device hot path ------------------------------------------------------
    def _torch_dtype(self):
        """Type of queries and of the K/V rows handed in (bf16 for int8 / fp8 pools)."""
        import torch
        return torch.bfloat16 if self.dtype in ("bf16", "int8", "fp8") else torch.float32

    # -- size checks: the C ABI cannot see device array sizes, so a short table,
    # kv_lens or row buffer would be read past its end by the kernels --------
    def _attn_sizes(self, q, block_tables, kv_lens, out, dims):
        """(B, H, d, max_blocks) of an attention call, checked against the pool
        and against each other."""
        if q.dim() != dims:
            raise ValueError(f"q must have {dims} dimensions, got shape {tuple(q.shape)}")
        B, H, d = int(q.shape[0]), int(q.shape[-2]), int(q.shape[-1])
        if d != self.head_dim:
            raise ValueError(f"q head_dim {d} != pool head_dim {self.head_dim}")
        if H % self.num_kv_heads:
            raise ValueError(f"num_heads {H} is not a multiple of num_kv_heads "
                             f"{self.num_kv_heads}")
        if block_tables.dim() != 2 or int(block_tables.shape[0]) < B:
            raise ValueError(f"block_tables must be [>= {B}, max_blocks], got "
                             f"{tuple(block_tables.shape)}")
        if kv_lens.numel() < B:
            raise ValueError(f"kv_lens needs {B} entries, got {kv_lens.numel()}")
        if out is not None and tuple(out.shape) != tuple(q.shape):
            raise ValueError(f"out must have shape {tuple(q.shape)}, got {tuple(out.shape)}")
        return B, H, d, int(block_tables.shape[1])

    def _row_sizes(self, key, value, n):
        """key / value must be [n, num_kv_heads, head_dim]."""
        want = (n, self.num_kv_heads, self.head_dim)
        for name, t in (("key", key), ("value", value)):
            if t is None or tuple(t.shape) != want:
                raise ValueError(f"{name} must have shape {want}, got "
                                 f"{None if t is None else tuple(t.shape)}")

    def append_kv(self, seqs, n_new, key, value, stream=None, return_slots=False):
        """Plan + copy-on-write + reshape_and_cache.  key/value [T, Hkv, d] CUDA."""
        seqs_a, sp = _i32(seqs)
        n_a, np_ = _i32(n_new)
        T = int(np.maximum(n_a, 0).sum())
        if T > 0:
            self._row_sizes(key, value, T)
        dt = self._torch_dtype()
        slots = np.zeros(max(T, 1), np.int64) if return_slots else None
        _check(lib().pa_append_kv(self._h, sp, np_, len(seqs_a),
                                  _dev_ptr(key, dt, "key"), _dev_ptr(value, dt, "value"),
                                  slots.ctypes.data_as(_PI64) if return_slots else None,
                                  _stream(stream)), "pa_append_kv")
        return slots[:T].tolist() if return_slots else None

    def reshape_and_cache(self, key, value, slot_mapping, stream=None):
        import torch
        self._row_sizes(key, value, int(slot_mapping.numel()))
        dt = self._torch_dtype()
        _check(lib().pa_reshape_and_cache(self._h, _dev_ptr(key, dt, "key"),
                                          _dev_ptr(value, dt, "value"),
                                          _dev_ptr(slot_mapping, torch.int64, "slot_mapping"),
                                          int(slot_mapping.numel()), _stream(stream)),
               "pa_reshape_and_cache")

    def cow_copy(self, src, dst, stream=None):
        import torch
        if src.numel() != dst.numel():
            raise ValueError(f"src and dst must pair up: {src.numel()} vs {dst.numel()}")
        _check(lib().pa_cow_copy(self._h, _dev_ptr(src, torch.int32, "src"),
                                 _dev_ptr(dst, torch.int32, "dst"), int(src.numel()),
                                 _stream(stream)), "pa_cow_copy")

    def decode_workspace_bytes(self, batch, num_heads, max_blocks, partition_tokens=0):
        return int(lib().pa_decode_workspace_bytes(self._h, batch, num_heads, max_blocks,
                                                   partition_tokens))

    def decode(self, q, block_tables, kv_lens, out=None, scale=None, partition_tokens=0,
               workspace=None, stream=None):
        """q [B, H, d] CUDA (pool dtype) -> out [B, H, d] float32."""
        import torch
        B, H, d, MB = self._attn_sizes(q, block_tables, kv_lens, out, 3)
        if out is None:
            out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
        scale = 1.0 / math.sqrt(self.head_dim) if scale is None else scale
        need = self.decode_workspace_bytes(B, H, MB, partition_tokens)
        if need and workspace is None:
            if self._ws is None or self._ws.numel() < need:
                self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            workspace = self._ws
        wp = _dev_ptr(workspace, None, "workspace") if need else None
        _check(lib().pa_decode(self._h, _dev_ptr(q, self._torch_dtype(), "q"), B, H,
                               _dev_ptr(block_tables, torch.int32, "block_tables"), MB,
                               _dev_ptr(kv_lens, torch.int32, "kv_lens"), float(scale),
                               int(partition_tokens), wp,
                               workspace.numel() if need else 0,
                               _dev_ptr(out, torch.float32, "out"), _stream(stream)),
               "pa_decode")
        return out

    def decode_window(self, q, block_tables, kv_lens, window, sinks=0, out=None, scale=None,
                      partition_tokens=0, workspace=None, stream=None):
        """Decode over a sink + recent window: key j visible iff j < sinks or
        j >= kv_len - window."""
        import torch
        B, H, d, MB = self._attn_sizes(q, block_tables, kv_lens, out, 3)
        if out is None:
            out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
        scale = 1.0 / math.sqrt(self.head_dim) if scale is None else scale
        need = int(lib().pa_decode_window_workspace_bytes(self._h, B, H, MB, int(window),
                                                          int(sinks), int(partition_tokens)))
        if need and workspace is None:
            if self._ws is None or self._ws.numel() < need:
                self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            workspace = self._ws
        wp = _dev_ptr(workspace, None, "workspace") if need else None
        _check(lib().pa_decode_window(self._h, _dev_ptr(q, self._torch_dtype(), "q"), B, H,
                                      _dev_ptr(block_tables, torch.int32, "block_tables"), MB,
                                      _dev_ptr(kv_lens, torch.int32, "kv_lens"), float(scale),
                                      int(window), int(sinks), int(partition_tokens), wp,
                                      workspace.numel() if need else 0,
                                      _dev_ptr(out, torch.float32, "out"), _stream(stream)),
               "pa_decode_window")
        return out

    def decode_window_append(self, q, key, value, slot_mapping, block_tables, kv_lens, window,
                             sinks=0, out=None, scale=None, partition_tokens=0, workspace=None,
                             stream=None):
        """decode_append over a sink + recent window: write each sequence's
        new token, then decode with key j visible iff j < sinks or
        j >= kv_len - window."""
        import torch
        B, H, d, MB = self._attn_sizes(q, block_tables, kv_lens, out, 3)
        self._row_sizes(key, value, B)
        if slot_mapping.numel() < B:
            raise ValueError(f"slot_mapping needs {B} entries, got {slot_mapping.numel()}")
        if out is None:
            out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
        scale = 1.0 / math.sqrt(self.head_dim) if scale is None else scale
        need = int(lib().pa_decode_window_workspace_bytes(self._h, B, H, MB, int(window),
                                                          int(sinks), int(partition_tokens)))
        if need and workspace is None:
            if self._ws is None or self._ws.numel() < need:
                self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            workspace = self._ws
        wp = _dev_ptr(workspace, None, "workspace") if need else None
        dt = self._torch_dtype()
        _check(lib().pa_decode_window_append(
            self._h, _dev_ptr(q, dt, "q"), _dev_ptr(key, dt, "key"), _dev_ptr(value, dt, "value"),
            _dev_ptr(slot_mapping, torch.int64, "slot_mapping"), B, H,
            _dev_ptr(block_tables, torch.int32, "block_tables"), MB,
            _dev_ptr(kv_lens, torch.int32, "kv_lens"), float(scale), int(window), int(sinks),
            int(partition_tokens), wp, workspace.numel() if need else 0,
            _dev_ptr(out, torch.float32, "out"), _stream(stream)), "pa_decode_window_append")
        return out

    def decode_append(self, q, key, value, slot_mapping, block_tables, kv_lens, out=None,
                      scale=None, partition_tokens=0, workspace=None, stream=None):
        """Fused step: write each sequence's new token (key/value [B, Hkv, d]
        at slot_mapping [B] int64) and decode q [B, H, d] over kv_lens."""
        import torch
        B, H, d, MB = self._attn_sizes(q, block_tables, kv_lens, out, 3)
        self._row_sizes(key, value, B)
        if slot_mapping.numel() < B:
            raise ValueError(f"slot_mapping needs {B} entries, got {slot_mapping.numel()}")
        if out is None:
            out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
        scale = 1.0 / math.sqrt(self.head_dim) if scale is None else scale
        need = self.decode_workspace_bytes(B, H, MB, partition_tokens)
        if need and workspace is None:
            if self._ws is None or self._ws.numel() < need:
                self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
            workspace = self._ws
        wp = _dev_ptr(workspace, None, "workspace") if need else None
        dt = self._torch_dtype()
        _check(lib().pa_decode_append(self._h, _dev_ptr(q, dt, "q"), _dev_ptr(key, dt, "key"),
                                      _dev_ptr(value, dt, "value"),
                                      _dev_ptr(slot_mapping, torch.int64, "slot_mapping"), B, H,
                                      _dev_ptr(block_tables, torch.int32, "block_tables"), MB,
                                      _dev_ptr(kv_lens, torch.int32, "kv_lens"), float(scale),
                                      int(partition_tokens), wp,
                                      workspace.numel() if need else 0,
                                      _dev_ptr(out, torch.float32, "out"), _stream(stream)),
               "pa_decode_append")
        return out

    def prefill_chunk(self, q, block_tables, kv_lens, out=None, scale=None, stream=None,
                      max_kv_splits=0):
        """q [B, q_tokens, H, d] CUDA (pool dtype) -> out float32, same shape.

        max_kv_splits: 0 = split the last wave's query tiles over their keys
        as the library chooses, 1 = never split, n = at most n parts."""
        import torch
        B, H, d, MB = self._attn_sizes(q, block_tables, kv_lens, out, 4)
        T = int(q.shape[1])
        if out is None:
            out = torch.empty((B, T, H, d), dtype=torch.float32, device=q.device)
        scale = 1.0 / math.sqrt(self.head_dim) if scale is None else scale
        _check(lib().pa_prefill_chunk(self._h, _dev_ptr(q, self._torch_dtype(), "q"), B, T, H,
                                      _dev_ptr(block_tables, torch.int32, "block_tables"), MB,
                                      _dev_ptr(kv_lens, torch.int32, "kv_lens"), float(scale),
                                      int(max_kv_splits), _dev_ptr(out, torch.float32, "out"),
                                      _stream(stream)),
               "pa_prefill_chunk")
        return out

    def get_error(self):
        """Synchronise; return and clear the device error bits (0 = none)."""
        code = C.c_int32()
        r = lib().pa_get_error(self._h, C.byref(code))
        if r not in (0, 6):
            raise PAError(r, "pa_get_error")
        return code.value

    def decode_path(self, num_heads):
        return int(lib().pa_decode_path(self._h, num_heads))

    def prefill_path(self, num_heads):
        return int(lib().pa_prefill_path(self._h, num_heads))


def _host_ptr(t, dtype, shape, name):
    """Address of a contiguous CPU tensor of the given dtype and shape."""
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous() or t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")
    return C.c_void_p(t.data_ptr())


class Batch:
    """A prepared decode batch (pa_batch_*): fixed sequences of ``pool``
    whose every step appends one token and decodes, from host buffers, in one
    C call.  ``step`` queues the work; ``sync`` waits for the outputs."""

    def __init__(self, pool, seqs, num_heads, max_blocks, partition_tokens=0):
        self.pool = pool
        self.seqs = [int(s) for s in seqs]
        self.num_heads, self.max_blocks = int(num_heads), int(max_blocks)
        seqs_a, sp = _i32(self.seqs)
        h = C.c_void_p()
        _check(lib().pa_batch_create(pool.handle, sp, len(seqs_a), self.num_heads,
                                     self.max_blocks, int(partition_tokens), C.byref(h)),
               "pa_batch_create")
        self._h = h

    def step(self, q, key, value, out, scale=None, stream=None):
        """q [n, H, d], key / value [n, Hkv, d] (pool dtype; bf16 for int8 /
        fp8 pools) and out [n, H, d] float32: pinned CPU tensors."""
        import torch
        p = self.pool
        n, d = len(self.seqs), p.head_dim
        dt = p._torch_dtype()
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        _check(lib().pa_batch_step(
            self._h, _host_ptr(q, dt, (n, self.num_heads, d), "q"),
            _host_ptr(key, dt, (n, p.num_kv_heads, d), "key"),
            _host_ptr(value, dt, (n, p.num_kv_heads, d), "value"), float(scale),
            _host_ptr(out, torch.float32, (n, self.num_heads, d), "out"), _stream(stream)),
            "pa_batch_step")

    def rollback(self):
        _check(lib().pa_batch_rollback(self._h), "pa_batch_rollback")

    def set_window(self, window, sinks=0):
        """Later steps decode over a sink + recent window (window 0: full)."""
        _check(lib().pa_batch_set_window(self._h, int(window), int(sinks)),
               "pa_batch_set_window")

    def sync(self):
        _check(lib().pa_batch_sync(self._h), "pa_batch_sync")

    def close(self):
        if getattr(self, "_h", None):
            lib().pa_batch_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
