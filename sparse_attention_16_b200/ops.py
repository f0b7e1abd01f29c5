"""ctypes binding of libdsa.so (include/dsa.h), argument marshalling only.

Each function takes torch tensors (device memory owned by the caller), checks
dtypes/shapes, and passes raw pointers and sizes to the C ABI on the current
torch stream.  All computation happens in the library's CUDA kernels; if the
library is missing or fails to load, every call raises - there is no CPU path.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_CUDA",
          4: "DSA_ERR_DEVICE_CHECK", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_WORKSPACE"}
DEVERR_BAD_INDEX, DEVERR_BAD_SEQ, DEVERR_MIXED_GROUP, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8

SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)

# Every symbol include/dsa.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float


class LayerArgs(ctypes.Structure):
    """Mirror of ``dsa_layer_args``."""

    _fields_ = [("q_nope", _P), ("q_pe", _P), ("qmul", _P), ("cache", _P), ("ld_c", _I32),
                ("d_rope", _I32), ("out", _P), ("lse", _P), ("out_f32", _I32), ("cache_fp8", _I32)]


class DeviceProps(ctypes.Structure):
    """Mirror of ``dsa_device_props``."""

    _fields_ = [("sms", _I32), ("max_clusters", _I32 * 9)]


class AttendPlan(ctypes.Structure):
    """Mirror of ``dsa_attend_plan``."""

    _fields_ = [("n_split", _I32), ("rows_per_split", _I32), ("merge", _I32), ("reserved", _I32),
                ("workspace_bytes", _SZ)]


class ForwardPlan(ctypes.Structure):
    """Mirror of ``dsa_forward_plan``."""

    _fields_ = [("chunk", _I32), ("n_chunks", _I32), ("last_chunk", _I32), ("attend_partials", _I32),
                ("idx_offset", _SZ), ("count_offset", _SZ), ("attend_offset", _SZ), ("attend_bytes", _SZ),
                ("hist_offset", _SZ), ("topk_offset", _SZ), ("topk_bytes", _SZ), ("scores_offset", _SZ),
                ("end", _SZ)]


SIGNATURES = {
    "dsa_index_scores": (_I32, [_P, _P, _P, _I64, _P, _I32, _P, _P, _I32, _I32, _P, _I64, _P, _P]),
    "dsa_index_scores_fp8": (_I32, [_P, _P, _P, _P, _P, _I64, _P, _I32, _P, _P, _I32, _I32, _P, _I64, _P, _P]),
    "dsa_topk_workspace_size": (_SZ, [_I32, _I64, _I32]),
    "dsa_topk": (_I32, [_P, _I64, _P, _I32, _I32, _P, _P, _P, _P, _SZ, _P]),
    "sparse_mla_workspace_size": (_SZ, [_I32, _I32]),
    "sparse_mla_attend": (_I32, [_P, _P, _P, _F, _P, _I64, _I32, _I32, _P, _I32, _P, _P, _P, _P, _I32,
                                 _I32, _P, _P, _P, _SZ, _P]),
    "sparse_mla_attend_noalloc": (_I32, [_P, _P, _P, _F, _P, _I64, _I32, _I32, _P, _I32, _P, _P, _P, _P,
                                         _I32, _I32, _P, _P, _P]),
    "sparse_mla_layers_workspace_size": (_SZ, [_I32, _I32, _I32]),
    "sparse_mla_attend_layers": (_I32, [_I32, ctypes.POINTER(LayerArgs), _F, _I64, _P, _I32, _P, _P, _P, _P,
                                        _I32, _I32, _P, _SZ, _P]),
    "dsa_forward_workspace_size": (_SZ, [_I32, _I64, _I32, _I32, _I32]),
    "dsa_sparse_mla_forward": (_I32, [_P, _P, _P, _I64, _P, _I32, _P, _P, _I32, _I32, _I64, _I32,
                                      ctypes.POINTER(LayerArgs), _F, _I32, _P, _P, _P, _SZ, _P]),
    "dsa_topk_export": (_I32, [_P, _I64, _P, _P, _I32, _I32, _I64, _P, _P, _P]),
    "dsa_topk_merge": (_I32, [_P, _P, _I32, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P]),
    "dsa_lse_combine": (_I32, [_P, _P, _I32, _I32, _P, _P, _P]),
    "dsa_get_device_props": (_I32, [ctypes.POINTER(DeviceProps)]),
    "dsa_plan_attend": (_I32, [_I32, _I32, _I32, _I32, ctypes.POINTER(DeviceProps), ctypes.POINTER(AttendPlan)]),
    "dsa_plan_forward": (_I32, [_I32, _I64, _I32, _I32, _I32, _I32, _I32, _SZ, ctypes.POINTER(DeviceProps),
                                ctypes.POINTER(ForwardPlan)]),
    "dsa_set_fault_test": (_I32, [ctypes.c_uint64, _I32]),
    "dsa_sparse_mla_forward_fp8": (_I32, [_P, _P, _P, _P, _P, _I64, _P, _I32, _P, _P, _I32, _I32, _I64, _I32,
                                          ctypes.POINTER(LayerArgs), _F, _I32, _P, _P, _P, _SZ, _P]),
    "dsa_check_errors": (_I32, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "dsa_launch_count": (ctypes.c_uint64, []),
    "dsa_last_error": (ctypes.c_char_p, []),
    "dsa_version": (_I32, []),
}

_lib = None


class DSAError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH):
    """Loads libdsa.so once and declares every exported function."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m sparse_attention_16_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status):
    if status != DSA_OK:
        raise DSAError(status, load_library().dsa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


# ----------------------------------------------------------------- calls

def index_scores(q_idx, w, k_idx, seq_row_start, q_seq, q_pos, scores, q_group=1, stream=None, hist=None):
    """I[t, s] into ``scores`` [T, ld] (see dsa_index_scores); with ``hist`` (uint32 [T, 2048],
    decode groups only) also the score histogram the top-k's histogram path uses."""
    T = q_idx.shape[0]
    _need(q_idx, torch.bfloat16, (T, 32, 128), "q_idx")
    _need(w, torch.float32, (T, 32), "w")
    _need(k_idx, torch.bfloat16, None, "k_idx")
    _need(seq_row_start, torch.int64, None, "seq_row_start")
    _need(q_seq, torch.int32, (T,), "q_seq")
    _need(q_pos, torch.int32, (T,), "q_pos")
    _need(scores, torch.float32, None, "scores")
    if hist is not None:
        _need(hist, torch.int32, (T, 2048), "hist")
    lib = load_library()
    _check(lib.dsa_index_scores(_ptr(q_idx), _ptr(w), _ptr(k_idx), k_idx.shape[0], _ptr(seq_row_start),
                                seq_row_start.shape[0], _ptr(q_seq), _ptr(q_pos), T, q_group,
                                _ptr(scores), scores.shape[1], _ptr(hist), _stream(stream)))
    return scores


def _codes(t, shape, name):
    """E4M3 codes as torch.float8_e4m3fn or their uint8 bytes."""
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    _need(t, torch.uint8, shape, name)
    return t


def index_scores_fp8(q8, q_scale, w, k8, k_scale, seq_row_start, q_seq, q_pos, scores, q_group=1,
                     stream=None, hist=None):
    """I[t, s] on FP8 (E4M3) keys and queries with per-row scales into ``scores``
    [T, ld] (see dsa_index_scores_fp8)."""
    T = q8.shape[0]
    q8 = _codes(q8, (T, 32, 128), "q8")
    k8 = _codes(k8, None, "k8")
    _need(q_scale, torch.float32, (T, 32), "q_scale")
    _need(w, torch.float32, (T, 32), "w")
    _need(k_scale, torch.float32, (k8.shape[0],), "k_scale")
    _need(seq_row_start, torch.int64, None, "seq_row_start")
    _need(q_seq, torch.int32, (T,), "q_seq")
    _need(q_pos, torch.int32, (T,), "q_pos")
    _need(scores, torch.float32, None, "scores")
    if hist is not None:
        _need(hist, torch.int32, (T, 2048), "hist")
    lib = load_library()
    _check(lib.dsa_index_scores_fp8(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), k8.shape[0],
                                    _ptr(seq_row_start), seq_row_start.shape[0], _ptr(q_seq), _ptr(q_pos), T,
                                    q_group, _ptr(scores), scores.shape[1], _ptr(hist), _stream(stream)))
    return scores


def topk_workspace_bytes(T, ld, k):
    return int(load_library().dsa_topk_workspace_size(T, ld, k))


def topk(scores, q_pos, k, idx, count, stream=None, hist=None, ws=None):
    """Top-k positions per query into ``idx`` [T, k] and ``count`` [T] (see dsa_topk); with the
    indexer's ``hist`` the first pass is skipped (a workspace is then needed)."""
    T = scores.shape[0]
    _need(scores, torch.float32, None, "scores")
    _need(q_pos, torch.int32, (T,), "q_pos")
    _need(idx, torch.int32, (T, k), "idx")
    _need(count, torch.int32, (T,), "count")
    if hist is not None:
        _need(hist, torch.int32, (T, 2048), "hist")
        if ws is None:
            ws = workspace(topk_workspace_bytes(T, scores.shape[1], k), scores.device)
    lib = load_library()
    _check(lib.dsa_topk(_ptr(scores), scores.shape[1], _ptr(q_pos), T, k, _ptr(idx), _ptr(count), _ptr(hist),
                        _ptr(ws) if hist is not None else None, ws.numel() if hist is not None else 0,
                        _stream(stream)))
    return idx, count


def attend_workspace_bytes(T, k):
    return int(load_library().sparse_mla_workspace_size(T, k))


def forward_workspace_bytes(T, ld, k, q_group=1, n_layers=1):
    return int(load_library().dsa_forward_workspace_size(T, ld, k, q_group, n_layers))


def device_props():
    """SM count and attention cluster residency of the current device (dsa_get_device_props)."""
    out = DeviceProps()
    _check(load_library().dsa_get_device_props(ctypes.byref(out)))
    return out


def make_props(sms, max_clusters):
    """A DeviceProps for planning without a GPU: max_clusters maps size c (2..8) to resident clusters."""
    d = DeviceProps()
    d.sms = sms
    for c, n in dict(max_clusters).items():
        d.max_clusters[c] = n
    return d


def plan_attend(T, n_layers=1, k=2048, props=None, allow_partials=True):
    """How the attention splits T queries x n_layers layers (dsa_plan_attend)."""
    out = AttendPlan()
    _check(load_library().dsa_plan_attend(T, n_layers, k, int(bool(allow_partials)),
                                          ctypes.byref(props) if props is not None else None, ctypes.byref(out)))
    return out


def plan_forward(T, ld, k, q_group, n_layers, has_idx_out, has_count_out, ws_bytes, props=None):
    """Chunking and workspace layout of dsa_sparse_mla_forward (dsa_plan_forward); raises
    DSAError(DSA_ERR_WORKSPACE) when nothing fits."""
    out = ForwardPlan()
    _check(load_library().dsa_plan_forward(T, ld, k, q_group, n_layers, int(bool(has_idx_out)),
                                           int(bool(has_count_out)), ws_bytes,
                                           ctypes.byref(props) if props is not None else None, ctypes.byref(out)))
    return out


def set_fault_test(wait_limit_ns=0, stall_tile=-1):
    """Testing hook of the attention kernel's timeout path (dsa_set_fault_test); (0, -1) = off."""
    _check(load_library().dsa_set_fault_test(int(wait_limit_ns), int(stall_tile)))


def workspace(nbytes, device):
    """A 256-byte aligned uint8 device buffer (torch allocations are 512-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def sparse_mla_attend(q_nope, q_pe, qmul, cache, d_rope, seq_row_start, q_seq, idx, count, out,
                      lse=None, softmax_scale=SOFTMAX_SCALE, ws=None, stream=None, q_pos=None):
    """Absorbed sparse MLA into ``out`` [T, 64, 512] bf16 (see sparse_mla_attend)."""
    T = q_nope.shape[0]
    k = idx.shape[1]
    _need(q_nope, torch.bfloat16, (T, 64, 512), "q_nope")
    if d_rope:
        _need(q_pe, torch.bfloat16, (T, 64, d_rope), "q_pe")
    _need(qmul, torch.float32, (T, 64), "qmul")
    _need(cache, torch.bfloat16, None, "cache")
    _need(idx, torch.int32, (T, k), "idx")
    _need(count, torch.int32, (T,), "count")
    _need(out, torch.bfloat16, (T, 64, 512), "out")
    if lse is not None:
        _need(lse, torch.float32, (T, 64), "lse")
    lib = load_library()
    need = attend_workspace_bytes(T, k)
    if ws is None and need > 0:
        ws = workspace(need, q_nope.device)
    if q_pos is not None:
        _need(q_pos, torch.int32, (T,), "q_pos")
    _check(lib.sparse_mla_attend(_ptr(q_nope), _ptr(q_pe) if d_rope else None, _ptr(qmul),
                                 float(softmax_scale), _ptr(cache), cache.shape[0], cache.shape[1],
                                 d_rope, _ptr(seq_row_start), seq_row_start.shape[0], _ptr(q_seq), _ptr(q_pos),
                                 _ptr(idx), _ptr(count), T, k, _ptr(out), _ptr(lse), _ptr(ws),
                                 0 if ws is None else ws.numel(), _stream(stream)))
    return out, lse


def sparse_mla_attend_noalloc(q_nope, q_pe, qmul, cache, d_rope, seq_row_start, q_seq, idx, count,
                              out, lse=None, softmax_scale=SOFTMAX_SCALE, stream=None, q_pos=None):
    """Same as sparse_mla_attend without a workspace, for callers that may not
    allocate device memory: the library's fixed scratch array holds the split
    partials (see sparse_mla_attend_noalloc in include/dsa.h for the limit and
    the rule that overlapping calls must be serialized)."""
    T = q_nope.shape[0]
    k = idx.shape[1]
    _need(q_nope, torch.bfloat16, (T, 64, 512), "q_nope")
    if d_rope:
        _need(q_pe, torch.bfloat16, (T, 64, d_rope), "q_pe")
    _need(qmul, torch.float32, (T, 64), "qmul")
    _need(cache, torch.bfloat16, None, "cache")
    _need(idx, torch.int32, (T, k), "idx")
    _need(count, torch.int32, (T,), "count")
    _need(out, torch.bfloat16, (T, 64, 512), "out")
    if lse is not None:
        _need(lse, torch.float32, (T, 64), "lse")
    lib = load_library()
    if q_pos is not None:
        _need(q_pos, torch.int32, (T,), "q_pos")
    _check(lib.sparse_mla_attend_noalloc(_ptr(q_nope), _ptr(q_pe) if d_rope else None, _ptr(qmul),
                                         float(softmax_scale), _ptr(cache), cache.shape[0], cache.shape[1],
                                         d_rope, _ptr(seq_row_start), seq_row_start.shape[0], _ptr(q_seq),
                                         _ptr(q_pos), _ptr(idx), _ptr(count), T, k, _ptr(out), _ptr(lse),
                                         _stream(stream)))
    return out, lse


def _layer_array(layers, T):
    arr = (LayerArgs * max(1, len(layers)))()
    for i, L in enumerate(layers):
        _need(L["q_nope"], torch.bfloat16, (T, 64, 512), f"layers[{i}].q_nope")
        if L["d_rope"]:
            _need(L["q_pe"], torch.bfloat16, (T, 64, L["d_rope"]), f"layers[{i}].q_pe")
        _need(L["qmul"], torch.float32, (T, 64), f"layers[{i}].qmul")
        fp8 = L["cache"].dtype == torch.uint8   # FP8 latent rows (E4M3 codes + block scales)
        _need(L["cache"], torch.uint8 if fp8 else torch.bfloat16, None, f"layers[{i}].cache")
        f32 = L["out"].dtype == torch.float32
        _need(L["out"], torch.float32 if f32 else torch.bfloat16, (T, 64, 512), f"layers[{i}].out")
        if L.get("lse") is not None:
            _need(L["lse"], torch.float32, (T, 64), f"layers[{i}].lse")
        arr[i] = LayerArgs(L["q_nope"].data_ptr(),
                           L["q_pe"].data_ptr() if L.get("q_pe") is not None else None,
                           L["qmul"].data_ptr(), L["cache"].data_ptr(), L["cache"].shape[1],
                           L["d_rope"], L["out"].data_ptr(),
                           L["lse"].data_ptr() if L.get("lse") is not None else None, int(f32), int(fp8))
    return arr


def layers_workspace_bytes(T, n_layers, k):
    return int(load_library().sparse_mla_layers_workspace_size(T, n_layers, k))


def sparse_mla_attend_layers(layers, n_rows, seq_row_start, q_seq, idx, count, q_pos=None,
                             softmax_scale=SOFTMAX_SCALE, ws=None, stream=None):
    """Attention of several layers over one shared selection (see sparse_mla_attend_layers).

    ``layers``: list of dicts with q_nope, q_pe (or None), qmul, cache, d_rope, out, lse (or None);
    every cache has ``n_rows`` rows.
    """
    T, k = idx.shape
    _need(idx, torch.int32, (T, k), "idx")
    _need(count, torch.int32, (T,), "count")
    _need(seq_row_start, torch.int64, None, "seq_row_start")
    _need(q_seq, torch.int32, (T,), "q_seq")
    if q_pos is not None:
        _need(q_pos, torch.int32, (T,), "q_pos")
    arr = _layer_array(layers, T)
    lib = load_library()
    need = layers_workspace_bytes(T, len(layers), k)
    if ws is None and need > 0:
        ws = workspace(need, idx.device)
    _check(lib.sparse_mla_attend_layers(len(layers), arr, float(softmax_scale), n_rows, _ptr(seq_row_start),
                                        seq_row_start.shape[0], _ptr(q_seq), _ptr(q_pos), _ptr(idx), _ptr(count),
                                        T, k, _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def sparse_mla_forward(q_idx, w, k_idx, seq_row_start, q_seq, q_pos, layers, ld, k=2048, q_group=1,
                       idx_out=None, count_out=None, softmax_scale=SOFTMAX_SCALE, ws=None,
                       stream=None):
    """Indexer + top-k once, then attention for every layer (see dsa_sparse_mla_forward).

    ``layers``: list of dicts with q_nope, q_pe (or None), qmul, cache, d_rope, out, lse (or None).
    """
    T = q_idx.shape[0]
    _need(q_idx, torch.bfloat16, (T, 32, 128), "q_idx")
    _need(w, torch.float32, (T, 32), "w")
    arr = _layer_array(layers, T)
    lib = load_library()
    if ws is None:
        ws = workspace(forward_workspace_bytes(T, ld, k, q_group, len(layers)), q_idx.device)
    _check(lib.dsa_sparse_mla_forward(_ptr(q_idx), _ptr(w), _ptr(k_idx), k_idx.shape[0],
                                      _ptr(seq_row_start), seq_row_start.shape[0], _ptr(q_seq),
                                      _ptr(q_pos), T, q_group, ld, len(layers), arr,
                                      float(softmax_scale), k, _ptr(idx_out), _ptr(count_out),
                                      _ptr(ws), ws.numel(), _stream(stream)))


def sparse_mla_forward_fp8(q8, q_scale, w, k8, k_scale, seq_row_start, q_seq, q_pos, layers, ld, k=2048,
                           q_group=1, idx_out=None, count_out=None, softmax_scale=SOFTMAX_SCALE, ws=None,
                           stream=None):
    """sparse_mla_forward with FP8 (E4M3) index keys and queries (see dsa_sparse_mla_forward_fp8)."""
    T = q8.shape[0]
    q8 = _codes(q8, (T, 32, 128), "q8")
    k8 = _codes(k8, None, "k8")
    _need(q_scale, torch.float32, (T, 32), "q_scale")
    _need(k_scale, torch.float32, (k8.shape[0],), "k_scale")
    _need(w, torch.float32, (T, 32), "w")
    arr = _layer_array(layers, T)
    lib = load_library()
    if ws is None:
        ws = workspace(forward_workspace_bytes(T, ld, k, q_group, len(layers)), q8.device)
    _check(lib.dsa_sparse_mla_forward_fp8(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), k8.shape[0],
                                          _ptr(seq_row_start), seq_row_start.shape[0], _ptr(q_seq), _ptr(q_pos), T,
                                          q_group, ld, len(layers), arr, float(softmax_scale), k, _ptr(idx_out),
                                          _ptr(count_out), _ptr(ws), ws.numel(), _stream(stream)))


# ----------------------------------------------------------------- context-parallel decode steps

def topk_export(scores, idx, count, pos_offset, out_score, out_pos, stream=None):
    """A rank's selection as (score, global position) exchange candidates (see dsa_topk_export)."""
    T, k = idx.shape
    _need(scores, torch.float32, None, "scores")
    _need(idx, torch.int32, (T, k), "idx")
    _need(count, torch.int32, (T,), "count")
    _need(out_score, torch.float32, (T, k), "out_score")
    _need(out_pos, torch.int32, (T, k), "out_pos")
    _check(load_library().dsa_topk_export(_ptr(scores), scores.shape[1], _ptr(idx), _ptr(count), T, k,
                                          int(pos_offset), _ptr(out_score), _ptr(out_pos), _stream(stream)))


def topk_merge(cand_score, cand_pos, k, count, idx_global=None, idx_local=None, count_local=None, shard=(0, 0),
               stream=None):
    """Global top-k from every rank's candidates [R, T, kr] (see dsa_topk_merge)."""
    R, T, kr = cand_pos.shape
    _need(cand_score, torch.float32, (R, T, kr), "cand_score")
    _need(cand_pos, torch.int32, (R, T, kr), "cand_pos")
    _need(count, torch.int32, (T,), "count")
    if idx_global is not None:
        _need(idx_global, torch.int32, (T, k), "idx_global")
    if idx_local is not None:
        _need(idx_local, torch.int32, (T, k), "idx_local")
        _need(count_local, torch.int32, (T,), "count_local")
    _check(load_library().dsa_topk_merge(_ptr(cand_score), _ptr(cand_pos), R, T, kr, k, int(shard[0]),
                                         int(shard[1]), _ptr(idx_global), _ptr(idx_local), _ptr(count_local),
                                         _ptr(count), _stream(stream)))


def lse_combine(o_parts, lse_parts, out, lse=None, stream=None):
    """Merge R partial attentions over disjoint parts of a selection (see dsa_lse_combine)."""
    R, T = lse_parts.shape[:2]
    _need(o_parts, torch.float32, (R, T, 64, 512), "o_parts")
    _need(lse_parts, torch.float32, (R, T, 64), "lse_parts")
    _need(out, torch.bfloat16, (T, 64, 512), "out")
    if lse is not None:
        _need(lse, torch.float32, (T, 64), "lse")
    _check(load_library().dsa_lse_combine(_ptr(o_parts), _ptr(lse_parts), R, T, _ptr(out), _ptr(lse),
                                          _stream(stream)))


def launch_count():
    """Kernels launched by the library in this process so far."""
    return int(load_library().dsa_launch_count())


def check_errors(stream=None):
    """Synchronizes and returns the device error word (raises DSAError if set)."""
    lib = load_library()
    bits = ctypes.c_uint32(0)
    st = lib.dsa_check_errors(_stream(stream), ctypes.byref(bits))
    if st != DSA_OK:
        raise DSAError(st, lib.dsa_last_error().decode() + f" (bits=0x{bits.value:x})")
    return bits.value
