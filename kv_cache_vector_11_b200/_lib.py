"""ctypes binding of libtq.so (argument marshalling only)."""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtq.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python kv_cache_vector_11_b200/build.py` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(_LIB_PATH)

FORMAT_VERSION = 1
STATUS_NORM_SATURATED = 1
STATUS_NONFINITE = 2
FMT_NORM_F32 = 1
FMT_NORM_CORRECTED = 2
FMT_GROUPED = 4

ROT_KINDS = {"wht": 0, "haar": 1, "gauss": 2}
DTYPES = {"f32": 0, "bf16": 1}

_c = ctypes
_vp = _c.c_void_p
_i32 = _c.c_int32
_i64 = _c.c_int64
_u64 = _c.c_uint64

_SIGS = {
    "tq_rotation_generate": (_i32, [_i32, _i32, _i32, _u64, _vp]),
    "tq_make_rotation": (_i32, [_i32, _i32, _i32, _u64, _c.POINTER(_vp)]),
    "tq_free_rotation": (None, [_vp]),
    "tq_rotation_copy_host": (_i32, [_vp, _vp]),
    "tq_rotation_info": (_i32, [_vp, _vp, _vp, _vp, _vp]),
    "tq_build_codebook": (_i32, [_i32, _i32, _vp, _vp]),
    "tq_code_words_per_row": (_i64, [_i32, _i32, _i32]),
    "tq_quantize_kv": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i64, _i32,
                               _vp, _vp, _vp, _vp, _vp, _vp]),
    "tq_quantize_kv_ex": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _c.c_uint32,
                                  _vp, _vp, _vp, _vp, _vp, _vp]),
    "tq_attn_logits_ex": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64,
                                  _i32, _c.c_uint32, _vp, _vp, _vp, _vp, _vp, _vp]),
    "tq_decode_attention_ex": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                       _i32, _i64, _i32, _c.c_uint32, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _c.c_float, _vp, _vp, _c.c_size_t, _vp]),
    "tq_attn_logits": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64,
                               _i32, _vp, _vp, _vp, _vp, _vp, _vp]),
    "tq_decode_workspace_size": (_c.c_size_t, [_i32, _i32, _i32, _i64, _i32]),
    "tq_decode_attention": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                    _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _c.c_float,
                                    _vp, _vp, _c.c_size_t, _vp]),
    "tq_decode_attention_static": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32,
                                           _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                           _c.c_float, _vp, _vp]),
    "tq_decode_append_paged": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                       _vp, _i32, _i32, _i32, _i32, _i64, _i32, _i32, _i32, _vp,
                                       _i32, _vp, _vp, _vp, _vp, _c.c_float, _vp, _vp, _c.c_size_t,
                                       _vp, _vp]),
    "tq_search_workspace_size": (_c.c_size_t, [_i32, _i64, _i32, _i32]),
    "tq_search_topk": (_i32, [_vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i64, _i32,
                              _vp, _vp, _vp, _c.c_size_t, _vp]),
    "tq_status_string": (_c.c_char_p, [_i32]),
    "tq_last_error": (_c.c_char_p, []),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib_path():
    return _LIB_PATH


def exported_symbols():
    """Names of the C entry points this binding uses (all declared in tq.h)."""
    return sorted(_SIGS)


class TQError(RuntimeError):
    def __init__(self, status, where):
        reason = _lib.tq_last_error().decode()
        super().__init__(f"{where}: {_lib.tq_status_string(status).decode()} ({reason})")
        self.status = status


def _check(status, where):
    if status != 0:
        raise TQError(status, where)


def _ptr(t):
    """Device or host pointer of a torch tensor / numpy array (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream_ptr(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _on(device):
    """Make ``device`` the current CUDA device for the C call: the library
    resolves per-device state (SM count, shared-memory limits, the static
    scratch address) through the current device."""
    import torch
    return torch.cuda.device(device)


def rotation_generate(kind, rows, cols, seed):
    """Dense float64 matrix of a seeded rotation / projection (host only)."""
    out = np.empty((rows, cols), dtype=np.float64)
    _check(_lib.tq_rotation_generate(ROT_KINDS[kind], rows, cols, seed, out.ctypes.data),
           "tq_rotation_generate")
    return out


def build_codebook(bits, block=32):
    """(centroids fp32 [2^bits], boundaries fp32 [2^bits - 1]) (host only)."""
    c = np.empty(1 << bits, dtype=np.float32)
    t = np.empty((1 << bits) - 1, dtype=np.float32)
    _check(_lib.tq_build_codebook(bits, block, c.ctypes.data, t.ctypes.data), "tq_build_codebook")
    return c, t


def code_words_per_row(bits, block, head_dim):
    return int(_lib.tq_code_words_per_row(bits, block, head_dim))


class Rotation:
    """Owning wrapper of a tq_rotation handle on the current CUDA device."""

    def __init__(self, kind, rows, cols, seed):
        h = _vp()
        _check(_lib.tq_make_rotation(ROT_KINDS[kind], rows, cols, seed, _c.byref(h)),
               "tq_make_rotation")
        self._h = h
        self.kind, self.rows, self.cols, self.seed = kind, rows, cols, seed

    @property
    def handle(self):
        return self._h

    def matrix(self):
        out = np.empty((self.rows, self.cols), dtype=np.float64)
        _check(_lib.tq_rotation_copy_host(self._h, out.ctypes.data), "tq_rotation_copy_host")
        return out

    def info(self):
        kind, rows, cols, seed = _i32(), _i32(), _i32(), _u64()
        _check(_lib.tq_rotation_info(self._h, _c.byref(kind), _c.byref(rows), _c.byref(cols),
                                     _c.byref(seed)), "tq_rotation_info")
        return kind.value, rows.value, cols.value, seed.value

    def close(self):
        if getattr(self, "_h", None):
            _lib.tq_free_rotation(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DTYPES["bf16"]
    if t.dtype == torch.float32:
        return DTYPES["f32"]
    raise TypeError(f"unsupported dtype {t.dtype}")


def _format(norm_f32, norm_correction, grouped=False):
    return ((FMT_NORM_F32 if norm_f32 else 0) | (FMT_NORM_CORRECTED if norm_correction else 0) |
            (FMT_GROUPED if grouped else 0))


def quantize_kv(rot, bits, centroids, boundaries, x, qjl=None, block=32, out=None,
                status=None, stream=None, norm_f32=False, norm_correction=False, grouped=False):
    """Quantize rows x [n_rows, head_dim] (bf16 or fp32, CUDA) with ``rot``.

    Returns dict(codes=uint32-as-int32 [n, W], norms=fp16 bits as int16 (fp32
    with ``norm_f32``) [n, d/block], and, with ``qjl``, signs [n, m/32], rnorm
    [n]).  ``out`` may supply those tensors to write into.  ``centroids`` and
    ``boundaries`` are the codebook of ``block``.  ``grouped`` writes the codes
    in the lane-grouped row order (TQ_FMT_GROUPED: value caches, bf16, d = 128).
    """
    import torch
    n, d = x.shape
    w = max(code_words_per_row(bits, block, d), 0)   # -1 for an unsupported block: the call rejects it
    dev = x.device
    if out is None:
        out = {"codes": torch.empty((n, w), dtype=torch.int32, device=dev),
               "norms": torch.empty((n, max(d // block, 0)),
                                    dtype=torch.float32 if norm_f32 else torch.int16, device=dev)}
        if qjl is not None:
            out["signs"] = torch.empty((n, qjl.rows // 32), dtype=torch.int32, device=dev)
            out["rnorm"] = torch.empty((n,), dtype=torch.int16, device=dev)
    c = np.ascontiguousarray(centroids, dtype=np.float32)
    t = np.ascontiguousarray(boundaries, dtype=np.float32)
    with _on(dev):
        _check(_lib.tq_quantize_kv_ex(
            rot.handle, bits, block, c.ctypes.data, t.ctypes.data,
            qjl.handle if qjl is not None else None,
            _ptr(x), _dtype_code(x), n, d, _format(norm_f32, norm_correction, grouped),
            _ptr(out["codes"]), _ptr(out["norms"]), _ptr(out.get("signs")), _ptr(out.get("rnorm")),
            _ptr(status), _stream_ptr(stream, dev)), "tq_quantize_kv_ex")
    return out


def attn_logits(rot, k_bits, k_centroids, q, k_codes, k_norms, n_kv_heads, ctx, qjl=None,
                qjl_signs=None, qjl_rnorm=None, block=32, logits=None, stream=None,
                norm_f32=False):
    """Raw scores [batch, n_q_heads, ctx] (fp32, CUDA) of q [batch, n_q_heads, d]."""
    import torch
    batch, n_q, d = q.shape
    if logits is None:
        logits = torch.empty((batch, n_q, ctx), dtype=torch.float32, device=q.device)
    c = np.ascontiguousarray(k_centroids, dtype=np.float32)
    with _on(q.device):
        _check(_lib.tq_attn_logits_ex(
            rot.handle, k_bits, block, c.ctypes.data, qjl.handle if qjl is not None else None,
            _ptr(q), _dtype_code(q), batch, n_q, n_kv_heads, ctx, d, _format(norm_f32, False),
            _ptr(k_codes), _ptr(k_norms), _ptr(qjl_signs), _ptr(qjl_rnorm), _ptr(logits),
            _stream_ptr(stream, q.device)), "tq_attn_logits_ex")
    return logits


def decode_workspace_size(batch, n_q_heads, n_kv_heads, ctx, head_dim):
    return int(_lib.tq_decode_workspace_size(batch, n_q_heads, n_kv_heads, ctx, head_dim))


def decode_attention(rot, k_bits, v_bits, k_centroids, v_centroids, q, k_codes, k_norms,
                     v_codes, v_norms, n_kv_heads, ctx, qjl=None, qjl_signs=None,
                     qjl_rnorm=None, scale=0.0, block=32, out=None, workspace=None,
                     stream=None, norm_f32=False, v_grouped=False):
    """Decode output [batch, n_q_heads, d] (fp32, CUDA).  ``v_grouped``: the
    value codes are in the lane-grouped row order (TQ_FMT_GROUPED)."""
    import torch
    batch, n_q, d = q.shape
    if out is None:
        out = torch.empty((batch, n_q, d), dtype=torch.float32, device=q.device)
    with _on(q.device):
        need = decode_workspace_size(batch, n_q, n_kv_heads, ctx, d)
        if workspace is None:
            workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
        kc = np.ascontiguousarray(k_centroids, dtype=np.float32)
        vc = np.ascontiguousarray(v_centroids, dtype=np.float32)
        _check(_lib.tq_decode_attention_ex(
            rot.handle, k_bits, v_bits, block, kc.ctypes.data, vc.ctypes.data,
            qjl.handle if qjl is not None else None,
            _ptr(q), _dtype_code(q), batch, n_q, n_kv_heads, ctx, d,
            _format(norm_f32, False, v_grouped),
            _ptr(k_codes), _ptr(k_norms), _ptr(qjl_signs), _ptr(qjl_rnorm),
            _ptr(v_codes), _ptr(v_norms), float(scale), _ptr(out),
            _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream_ptr(stream, q.device)), "tq_decode_attention_ex")
    return out


DECODE_STATIC_SCRATCH_BYTES = 16 << 20


def decode_attention_static(rot, k_bits, v_bits, k_centroids, v_centroids, q, k_codes, k_norms,
                            v_codes, v_norms, n_kv_heads, ctx, qjl=None, qjl_signs=None,
                            qjl_rnorm=None, scale=0.0, block=32, out=None, stream=None):
    """``decode_attention`` without a workspace, for callers that cannot
    allocate device memory on the call path (engine plugins that must not
    allocate while enqueueing, servers that hand out memory only from a
    pre-reserved arena, loops that must avoid cudaMalloc's implicit device
    synchronisation).  The split partials live in a fixed 16 MiB array inside
    the library; larger shapes raise TQError.  Calls that overlap on the GPU
    share that array and race, so issue them on one stream.  ``out`` may be
    passed in so the call itself allocates nothing."""
    import torch
    batch, n_q, d = q.shape
    if out is None:
        out = torch.empty((batch, n_q, d), dtype=torch.float32, device=q.device)
    kc = np.ascontiguousarray(k_centroids, dtype=np.float32)
    vc = np.ascontiguousarray(v_centroids, dtype=np.float32)
    with _on(q.device):
        _check(_lib.tq_decode_attention_static(
            rot.handle, k_bits, v_bits, block, kc.ctypes.data, vc.ctypes.data,
            qjl.handle if qjl is not None else None,
            _ptr(q), _dtype_code(q), batch, n_q, n_kv_heads, ctx, d,
            _ptr(k_codes), _ptr(k_norms), _ptr(qjl_signs), _ptr(qjl_rnorm),
            _ptr(v_codes), _ptr(v_norms), float(scale), _ptr(out),
            _stream_ptr(stream, q.device)), "tq_decode_attention_static")
    return out


def search_workspace_size(n_queries, n_db, head_dim, k):
    return int(_lib.tq_search_workspace_size(n_queries, n_db, head_dim, k))


def search_topk(rot, bits, centroids, q, db_codes, db_norms, k, block=32, workspace=None,
                stream=None):
    """Top-k maximum-inner-product search of queries q [n_q, head_dim] (bf16
    or fp32, CUDA) over packed database rows; returns (scores fp32 [n_q, k],
    rows int32 [n_q, k])."""
    import torch
    n_q, d = q.shape
    n_db = db_codes.shape[0]
    scores = torch.empty((n_q, k), dtype=torch.float32, device=q.device)
    rows = torch.empty((n_q, k), dtype=torch.int32, device=q.device)
    c = np.ascontiguousarray(centroids, dtype=np.float32)
    with _on(q.device):
        need = search_workspace_size(n_q, n_db, d, k)
        if workspace is None:
            workspace = torch.empty((max(need, 256),), dtype=torch.uint8, device=q.device)
        _check(_lib.tq_search_topk(
            rot.handle, bits, block, c.ctypes.data, _ptr(q), _dtype_code(q), n_q, d,
            _ptr(db_codes), _ptr(db_norms), n_db, k, _ptr(scores), _ptr(rows), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream_ptr(stream, q.device)),
            "tq_search_topk")
    return scores, rows


def decode_append_paged(rot, k_bits, v_bits, k_codebook, v_codebook, q, k_new, v_new, pages,
                        block_table, n_kv_heads, ctx, page_size, scale=0.0, out=None,
                        workspace=None, status=None, stream=None):
    """One decode step that first appends the step's token: k_new / v_new
    [batch, n_kv_heads, head_dim] are quantized into token ctx - 1 of the paged
    cache ``pages`` (dict of k_codes, k_norms, v_codes, v_norms, each
    [n_pages, n_kv_heads, page_size, ...] on the device) through
    ``block_table`` (int32 [batch, max_pages]); returns the attention output
    [batch, n_q_heads, head_dim] over tokens 0 .. ctx - 1.  ``k_codebook`` and
    ``v_codebook`` are (centroids, boundaries) pairs."""
    import torch
    batch, n_q, d = q.shape
    if out is None:
        out = torch.empty((batch, n_q, d), dtype=torch.float32, device=q.device)
    kc = np.ascontiguousarray(k_codebook[0], dtype=np.float32)
    kt = np.ascontiguousarray(k_codebook[1], dtype=np.float32)
    vc = np.ascontiguousarray(v_codebook[0], dtype=np.float32)
    vt = np.ascontiguousarray(v_codebook[1], dtype=np.float32)
    n_pages = pages["k_codes"].shape[0]
    with _on(q.device):
        need = decode_workspace_size(batch, n_q, n_kv_heads, ctx, d)
        if workspace is None:
            workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
        _check(_lib.tq_decode_append_paged(
            rot.handle, k_bits, v_bits, 32, kc.ctypes.data, kt.ctypes.data, vc.ctypes.data,
            vt.ctypes.data, _ptr(q), _dtype_code(q), _ptr(k_new), _ptr(v_new), _dtype_code(k_new),
            batch, n_q, n_kv_heads, ctx, d, page_size, n_pages, _ptr(block_table),
            block_table.shape[1], _ptr(pages["k_codes"]), _ptr(pages["k_norms"]),
            _ptr(pages["v_codes"]), _ptr(pages["v_norms"]), float(scale), _ptr(out),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
            _stream_ptr(stream, q.device)), "tq_decode_append_paged")
    return out
