"""ctypes binding of libwf (the C ABI in include/wf.h and include/wf_synth.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Functions keep the C names.  Tensors may be passed as torch
tensors (their data_ptr is used) or raw integer addresses; streams as
``torch.cuda.Stream`` or integer handles (``None`` = legacy default stream).
Loading fails loudly when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import struct
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwf.so")

WF_OK, WF_ERR_INVALID_ARG, WF_ERR_UNSUPPORTED, WF_ERR_ALIGNMENT, WF_ERR_CAPACITY, \
    WF_ERR_WORKSPACE, WF_ERR_CUDA, WF_ERR_DEVICE_TIMEOUT, WF_ERR_PLAN = range(9)
WF_F32, WF_BF16 = 0, 1
WF_MAX_INROUND = 16
WF_SYNTH_Q, WF_SYNTH_K, WF_SYNTH_V = 1, 2, 3
WF_FP8_BLOCK = 128
WF_ATTN_STATUS_BYTES = 256
WF_FP8_Q, WF_FP8_K = 0, 1

# exported symbols, in the order include/wf.h and include/wf_synth.h declare them
EXPORTS = ("wf_plan_bytes", "wf_plan_round", "wf_balance_units", "wf_rope3d_append", "wf_attn_workspace_bytes",
           "wf_attn_workspace_init", "wf_attn_workspace_status", "wf_chunk_causal_attn", "wf_rope3d_append_kv",
           "wf_chunk_causal_attn_rope",
           "wf_chunk_causal_attn_noalloc", "wf_attn_noalloc_status", "wf_quantize_fp8", "wf_chunk_causal_attn_fp8",
           "wf_status_string", "wf_version", "wf_synth_fill")


class WfError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)}")


class RoundDesc(ctypes.Structure):
    _fields_ = [
        ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("frame_h", ctypes.c_int32), ("frame_w", ctypes.c_int32),
        ("frames_per_chunk", ctypes.c_int32), ("cache_chunks", ctypes.c_int32),
        ("inround_chunks", ctypes.c_int32), ("pool_slots", ctypes.c_int32),
        ("n0", ctypes.c_int64),
        ("noise_t", ctypes.c_int32 * WF_MAX_INROUND),
        ("rope_pairs_t", ctypes.c_int32), ("rope_pairs_h", ctypes.c_int32), ("rope_pairs_w", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("dtype", ctypes.c_int32), ("num_ctas", ctypes.c_int32),
    ]


def make_desc(H, D, fh, fw, F, Wc, R, n0, noise_t: Sequence[int], *, S=0, pairs=(0, 0, 0),
              theta=10000.0, dtype=WF_BF16, num_ctas=0) -> RoundDesc:
    d = RoundDesc()
    d.num_heads, d.head_dim, d.frame_h, d.frame_w, d.frames_per_chunk = H, D, fh, fw, F
    d.cache_chunks, d.inround_chunks, d.pool_slots, d.n0 = Wc, R, S, n0
    for i, t in enumerate(noise_t):
        d.noise_t[i] = int(t)
    d.rope_pairs_t, d.rope_pairs_h, d.rope_pairs_w = pairs
    d.rope_theta, d.dtype, d.num_ctas = float(theta), int(dtype), int(num_ctas)
    return d


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libwf.so is not built ({LIB_PATH}); run "
                               "`python -m chunk_causal_attention_block_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
        dp = ctypes.POINTER(RoundDesc)
        L.wf_plan_bytes.argtypes, L.wf_plan_bytes.restype = [dp], sz
        L.wf_plan_round.argtypes, L.wf_plan_round.restype = [dp, vp, sz, vp, sz, vp], i32
        L.wf_balance_units.argtypes, L.wf_balance_units.restype = [vp, i32, i32, vp, vp], i32
        L.wf_rope3d_append.argtypes, L.wf_rope3d_append.restype = [vp] * 8 + [vp], i32
        L.wf_rope3d_append_kv.argtypes, L.wf_rope3d_append_kv.restype = [vp] * 6 + [vp], i32
        L.wf_chunk_causal_attn_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, sz, vp]
        L.wf_chunk_causal_attn_rope.restype = i32
        L.wf_attn_workspace_bytes.argtypes, L.wf_attn_workspace_bytes.restype = [vp], sz
        L.wf_attn_workspace_init.argtypes, L.wf_attn_workspace_init.restype = [vp, sz, vp], i32
        L.wf_attn_workspace_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
        L.wf_attn_workspace_status.restype = i32
        L.wf_chunk_causal_attn.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, sz, vp]
        L.wf_chunk_causal_attn.restype = i32
        L.wf_chunk_causal_attn_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp]
        L.wf_chunk_causal_attn_noalloc.restype = i32
        L.wf_attn_noalloc_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        L.wf_attn_noalloc_status.restype = i32
        L.wf_quantize_fp8.argtypes, L.wf_quantize_fp8.restype = [vp, vp, vp, vp, i32, vp], i32
        L.wf_chunk_causal_attn_fp8.argtypes = [vp] * 9 + [ctypes.c_float, vp, sz, vp]
        L.wf_chunk_causal_attn_fp8.restype = i32
        L.wf_status_string.argtypes, L.wf_status_string.restype = [i32], ctypes.c_char_p
        L.wf_version.argtypes, L.wf_version.restype = [], i32
        L.wf_synth_fill.argtypes = [vp, i32, u64, i32, i64, i64, i32, i32, i32, i32, i32, vp]
        L.wf_synth_fill.restype = i32
        _lib = L
    return _lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(code: int, where: str):
    if code != WF_OK:
        raise WfError(code, where)


def status_string(code: int) -> str:
    return lib().wf_status_string(code).decode()


wf_status_string = status_string


def wf_version() -> int:
    return lib().wf_version()


def wf_plan_bytes(desc: RoundDesc) -> int:
    return lib().wf_plan_bytes(ctypes.byref(desc))


def wf_plan_round(desc: RoundDesc, host_plan, dev_plan=None, stream=None, host_bytes=None, dev_bytes=None):
    hb = host_bytes if host_bytes is not None else _nbytes(host_plan)
    db = dev_bytes if dev_bytes is not None else (_nbytes(dev_plan) if dev_plan is not None else 0)
    _check(lib().wf_plan_round(ctypes.byref(desc), _ptr(host_plan), hb, _ptr(dev_plan), db, _stream(stream)),
           "wf_plan_round")


def wf_balance_units(costs: Sequence[int], bins: int):
    """Per bin, the item indices the library's work balancer assigns to it, in list order."""
    cost = np.ascontiguousarray(np.asarray(costs, dtype=np.int64).reshape(-1))
    start = np.zeros(bins + 1, dtype=np.int32)
    items = np.zeros(max(len(cost), 1), dtype=np.int32)
    _check(lib().wf_balance_units(cost.ctypes.data, len(cost), bins, start.ctypes.data, items.ctypes.data),
           "wf_balance_units")
    return [items[start[b]:start[b + 1]].tolist() for b in range(bins)]


def wf_rope3d_append(host_plan, dev_plan, q, k, v, q_rot, k_pool, v_pool, stream=None):
    _check(lib().wf_rope3d_append(_ptr(host_plan), _ptr(dev_plan), _ptr(q), _ptr(k), _ptr(v), _ptr(q_rot),
                                  _ptr(k_pool), _ptr(v_pool), _stream(stream)), "wf_rope3d_append")


def wf_rope3d_append_kv(host_plan, dev_plan, k, v, k_pool, v_pool, stream=None):
    _check(lib().wf_rope3d_append_kv(_ptr(host_plan), _ptr(dev_plan), _ptr(k), _ptr(v), _ptr(k_pool), _ptr(v_pool),
                                     _stream(stream)), "wf_rope3d_append_kv")


def wf_attn_workspace_bytes(host_plan) -> int:
    return lib().wf_attn_workspace_bytes(_ptr(host_plan))


def wf_attn_workspace_init(workspace, stream=None, nbytes=None):
    _check(lib().wf_attn_workspace_init(_ptr(workspace), nbytes or _nbytes(workspace), _stream(stream)),
           "wf_attn_workspace_init")


def wf_attn_workspace_status(workspace, stream=None):
    """Returns (status code, [code, where, block, thread]); synchronises `stream`."""
    detail = (ctypes.c_int32 * 4)()
    code = lib().wf_attn_workspace_status(_ptr(workspace), _stream(stream), detail)
    return code, list(detail)


def wf_chunk_causal_attn(host_plan, dev_plan, q_rot, k_pool, v_pool, out, lse=None, softmax_scale=0.0,
                         workspace=None, stream=None, workspace_bytes=None):
    wb = workspace_bytes if workspace_bytes is not None else _nbytes(workspace)
    _check(lib().wf_chunk_causal_attn(_ptr(host_plan), _ptr(dev_plan), _ptr(q_rot), _ptr(k_pool), _ptr(v_pool),
                                      _ptr(out), _ptr(lse), float(softmax_scale), _ptr(workspace), wb,
                                      _stream(stream)), "wf_chunk_causal_attn")


def wf_chunk_causal_attn_rope(host_plan, dev_plan, q, k_pool, v_pool, out, lse=None, softmax_scale=0.0,
                              workspace=None, stream=None, workspace_bytes=None):
    """wf_chunk_causal_attn from raw queries: the kernel applies Q's RoPE."""
    wb = workspace_bytes if workspace_bytes is not None else _nbytes(workspace)
    _check(lib().wf_chunk_causal_attn_rope(_ptr(host_plan), _ptr(dev_plan), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                           _ptr(out), _ptr(lse), float(softmax_scale), _ptr(workspace), wb,
                                           _stream(stream)), "wf_chunk_causal_attn_rope")


def wf_chunk_causal_attn_noalloc(host_plan, dev_plan, q_rot, k_pool, v_pool, out, lse=None, softmax_scale=0.0,
                                 stream=None):
    """wf_chunk_causal_attn without a caller workspace (library-held static scratch)."""
    _check(lib().wf_chunk_causal_attn_noalloc(_ptr(host_plan), _ptr(dev_plan), _ptr(q_rot), _ptr(k_pool),
                                              _ptr(v_pool), _ptr(out), _ptr(lse), float(softmax_scale),
                                              _stream(stream)), "wf_chunk_causal_attn_noalloc")


def wf_attn_noalloc_status(stream=None):
    """Device status of the last no-alloc call on the current device: (status code,
    [code, where, block, thread]); synchronises `stream`."""
    detail = (ctypes.c_int32 * 4)()
    code = lib().wf_attn_noalloc_status(_stream(stream), detail)
    return code, list(detail)



def wf_quantize_fp8(host_plan, src, dst8, scales, which, stream=None):
    _check(lib().wf_quantize_fp8(_ptr(host_plan), _ptr(src), _ptr(dst8), _ptr(scales), int(which), _stream(stream)),
           "wf_quantize_fp8")


def wf_chunk_causal_attn_fp8(host_plan, dev_plan, q8, q_scales, k8_pool, k_scales, v_pool, out, lse=None,
                             softmax_scale=0.0, workspace=None, stream=None, workspace_bytes=None):
    wb = workspace_bytes if workspace_bytes is not None else _nbytes(workspace)
    _check(lib().wf_chunk_causal_attn_fp8(_ptr(host_plan), _ptr(dev_plan), _ptr(q8), _ptr(q_scales), _ptr(k8_pool),
                                          _ptr(k_scales), _ptr(v_pool), _ptr(out), _ptr(lse), float(softmax_scale),
                                          _ptr(workspace), wb, _stream(stream)), "wf_chunk_causal_attn_fp8")

def wf_synth_fill(dst, dtype, seed, tensor, tag, n_first, nchunks, C, H, D, kscale=False, stream=None):
    _check(lib().wf_synth_fill(_ptr(dst), int(dtype), int(seed) & 0xFFFFFFFFFFFFFFFF, int(tensor), int(tag),
                               int(n_first), int(nchunks), int(C), int(H), int(D), int(bool(kscale)),
                               _stream(stream)), "wf_synth_fill")


def _nbytes(x) -> int:
    if x is None:
        return 0
    if isinstance(x, np.ndarray):
        return x.nbytes
    return x.numel() * x.element_size()


# --------------------------------------------------------------------------
# plan blob decoding (host copy), mirroring csrc/wf_plan.h
# --------------------------------------------------------------------------

_HDR = struct.Struct("<IIQ" + "i" * 20 + "qqd" + "Q" * 7 + "16i")
_CHUNK = struct.Struct("<q" + "i" * 12)
assert _HDR.size == 240 and _CHUNK.size == 56


def decode_plan(blob) -> dict:
    b = bytes(np.asarray(blob, dtype=np.uint8).reshape(-1).tobytes())
    v = _HDR.unpack_from(b, 0)
    names = ["magic", "version", "total_bytes", "H", "D", "fh", "fw", "F", "C", "Wc", "wc_eff", "R", "S",
             "dtype", "Pt", "Ph", "Pw", "num_ctas", "num_units", "q_pairs", "q_tiles", "max_key_tiles",
             "max_nvis", "n0", "first", "theta", "off_chunks", "off_vis", "off_rope_t", "off_rope_h",
             "off_rope_w", "off_units", "off_cta"]
    h = dict(zip(names, v[:len(names)]))
    h["noise_t"] = list(v[len(names):len(names) + h["R"]])
    chunks = []
    for i in range(h["R"]):
        c = _CHUNK.unpack_from(b, h["off_chunks"] + 56 * i)
        n, slot, noise, nvis, keys, s0, s1, l0, l1, t0, t1, kt, fb = c
        vis = np.frombuffer(b, dtype=np.int32, count=h["Wc"] + h["R"],
                            offset=h["off_vis"] + 4 * i * (h["Wc"] + h["R"]))
        chunks.append(dict(n=n, slot=slot, noise=noise, nvis=nvis, keys=keys, segs=[(s0, l0), (s1, l1)],
                           seg_tiles=[t0, t1], key_tiles=kt, frame_base=fb,
                           vis_slots=[int(x) for x in vis[:nvis]]))
    h["chunks"] = chunks

    def table(off, rows, P):
        a = np.frombuffer(b, dtype=np.float64, count=2 * rows * P, offset=off).reshape(rows, P, 2)
        return a[..., 0], a[..., 1]
    h["rope_t"] = table(h["off_rope_t"], h["R"] * h["F"], h["Pt"])
    h["rope_h"] = table(h["off_rope_h"], h["fh"], h["Ph"])
    h["rope_w"] = table(h["off_rope_w"], h["fw"], h["Pw"])
    cta = np.frombuffer(b, dtype=np.int32, count=h["num_ctas"] + 1, offset=h["off_cta"])
    units = np.frombuffer(b, dtype=np.int32, count=8 * h["num_units"], offset=h["off_units"]).reshape(-1, 8)
    # (chunk, head, pair, cost, part, parts, slot) per unit
    h["per_cta"] = [[tuple(int(x) for x in units[u][:7]) for u in range(cta[c], cta[c + 1])]
                    for c in range(h["num_ctas"])]
    h["key_parts"] = int(units[0][5]) if h["num_units"] else 1
    return h


def host_plan_buffer(desc: RoundDesc, pinned: bool = False):
    """A 16-byte-aligned host buffer (torch uint8, pinned if asked) for the plan of `desc`."""
    import torch
    n = wf_plan_bytes(desc)
    if n == 0:
        raise WfError(WF_ERR_INVALID_ARG, "wf_plan_bytes")
    return torch.empty(n, dtype=torch.uint8, pin_memory=pinned)
