"""ctypes binding of ``libsoup.so`` (the C ABI in ``include/soup.h``).

Argument marshalling only: every function takes PyTorch tensors (device
memory and streams come from PyTorch), passes their raw pointers and sizes to
the C entry point of the same name, and raises ``SoupError`` on a nonzero
status.  There is no fallback: if the library is missing, importing a function
raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsoup.so")

c_void_p, c_int32, c_int64, c_float, c_size_t = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                                  ctypes.c_float, ctypes.c_size_t)

SOUP_WEIGHT_NF4 = 0
SOUP_WEIGHT_BF16 = 1


class SoupError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


class SoupWeight(ctypes.Structure):
    _fields_ = [("kind", c_int32), ("out_features", c_int64), ("in_features", c_int64),
                ("codes", c_void_p), ("absmax", c_void_p), ("w", c_void_p)]


class LayerCfg(ctypes.Structure):
    _fields_ = [("hidden", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32), ("head_dim", c_int32),
                ("intermediate", c_int32), ("rank", c_int32), ("alpha", c_float), ("eps", c_float),
                ("theta", c_float), ("prefix_share", c_int32), ("prefix_len", c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("qkv", SoupWeight), ("o", SoupWeight), ("gate_up", SoupWeight), ("down", SoupWeight),
                ("norm1", c_void_p), ("norm2", c_void_p)]


class LayerLora(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("A_qkv", "B_qkv", "A_o", "B_o", "A_gu", "B_gu", "A_down", "B_down")]


class LayerGrads(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("dA_qkv", "dB_qkv", "dA_o", "dB_o", "dA_gu", "dB_gu", "dA_down",
                                        "dB_down")]


class StreamDesc(ctypes.Structure):
    _fields_ = [("n_layers", c_int32), ("layer_bytes", c_size_t), ("host_layers", ctypes.POINTER(c_void_p)),
                ("vocab_bytes", c_size_t), ("host_embed", c_void_p), ("host_head", c_void_p),
                ("n_buffers", c_int32), ("device_cap_bytes", c_size_t), ("reserve_bytes", c_size_t)]


class StreamStats(ctypes.Structure):
    _fields_ = [("copies", c_int64), ("reuses", c_int64), ("bytes_copied", c_size_t), ("arena_bytes", c_size_t),
                ("waits", c_int64), ("stall_ms", ctypes.c_double), ("copy_ms", ctypes.c_double)]


class DiskStats(ctypes.Structure):
    _fields_ = [("reads", c_int64), ("skipped", c_int64), ("acquires", c_int64), ("bytes_read", ctypes.c_uint64),
                ("read_ms", ctypes.c_double), ("wait_ms", ctypes.c_double), ("direct_files", c_int32)]


SOUP_DISK_PINNED, SOUP_DISK_DIRECT = 1, 2


class GemmProfile(ctypes.Structure):
    _fields_ = [("launches", c_int64), ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


GEMM_CLASSES = ("nf4_fwd", "nf4_bwd", "bf16", "lora_skinny", "nf4_dual")
# every class soup_profile_enable can time, in bit order: the GEMM classes,
# then attention (flops) and the memory-bound kernels (algorithmic bytes)
PROFILE_CLASSES = GEMM_CLASSES + ("attention", "rmsnorm", "splitk_reduce", "elementwise", "ce_rows", "adamw")
HBM_CLASSES = ("rmsnorm", "splitk_reduce", "elementwise", "ce_rows", "adamw")
PROFILE_ALL = (1 << len(PROFILE_CLASSES)) - 1

SOUP_ITEM_EMBED = -1
SOUP_ITEM_HEAD = -2

# name -> (restype, argtypes)
_SIGS = {
    "soup_last_error": (ctypes.c_char_p, []),
    "soup_device_error": (c_int32, [ctypes.POINTER(c_int32)]),
    "soup_launch_count": (c_int64, []),
    "soup_profile_enable": (c_int32, [c_int32]),
    "soup_profile_read": (c_int32, [ctypes.POINTER(GemmProfile), c_int32]),
    "soup_nf4_quantize": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p]),
    "soup_nf4_dequant": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
    "soup_lora_linear_fwd": (c_int32, [ctypes.POINTER(SoupWeight), c_void_p, c_void_p, c_int32, c_float,
                                       c_void_p, c_int64, c_void_p, c_void_p, c_void_p]),
    "soup_lora_linear_bwd_workspace": (c_size_t, [c_int64, c_int32, c_int64]),
    "soup_lora_linear_bwd": (c_int32, [ctypes.POINTER(SoupWeight), c_void_p, c_void_p, c_int32, c_float,
                                       c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_size_t, c_void_p]),
    "soup_lora_linear_bwd_noalloc_max_scratch": (c_size_t, []),
    "soup_lora_linear_bwd_noalloc": (c_int32, [ctypes.POINTER(SoupWeight), c_void_p, c_void_p, c_int32, c_float,
                                               c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                               c_void_p]),
    "soup_decoder_layer_workspace": (c_size_t, [ctypes.POINTER(LayerCfg), c_int64, c_int64]),
    "soup_decoder_layer_fwd": (c_int32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerLora),
                                         ctypes.POINTER(LayerCfg), c_void_p, c_int64, c_int64, c_void_p, c_int32,
                                         c_void_p, c_size_t, c_void_p]),
    "soup_decoder_layer_bwd": (c_int32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerLora),
                                         ctypes.POINTER(LayerCfg), c_void_p, c_void_p, c_int64, c_int64, c_void_p,
                                         ctypes.POINTER(LayerGrads), c_int32, c_void_p, c_size_t, c_void_p]),
    "soup_decoder_layer_keep_bytes": (c_size_t, [ctypes.POINTER(LayerCfg), c_int64, c_int64]),
    "soup_decoder_layer_fwd_keep": (c_int32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerLora),
                                              ctypes.POINTER(LayerCfg), c_void_p, c_int64, c_int64, c_void_p,
                                              c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "soup_decoder_layer_bwd_kept": (c_int32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerLora),
                                              ctypes.POINTER(LayerCfg), c_void_p, c_void_p, c_int64, c_int64,
                                              c_void_p, ctypes.POINTER(LayerGrads), c_int32, c_void_p, c_void_p,
                                              c_size_t, c_void_p]),
    "soup_decoder_layer_saved_bytes": (c_size_t, [ctypes.POINTER(LayerCfg), c_int64, c_int64]),
    "soup_decoder_layer_fwd_save": (c_int32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerLora),
                                              ctypes.POINTER(LayerCfg), c_void_p, c_int64, c_int64, c_void_p,
                                              c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "soup_decoder_layer_bwd_saved": (c_int32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerLora),
                                               ctypes.POINTER(LayerCfg), c_void_p, c_void_p, c_int64, c_int64,
                                               c_void_p, ctypes.POINTER(LayerGrads), c_int32, c_void_p, c_void_p,
                                               c_size_t, c_void_p]),
    "soup_stream_plan": (c_int32, [ctypes.POINTER(StreamDesc), ctypes.POINTER(c_void_p)]),
    "soup_stream_plan_free": (c_int32, [c_void_p]),
    "soup_stream_prefetch": (c_int32, [c_void_p, c_int32]),
    "soup_stream_prefetch_from": (c_int32, [c_void_p, c_int32, c_void_p, c_void_p]),
    "soup_stream_resident": (c_int32, [c_void_p, c_int32, ctypes.POINTER(c_int32)]),
    "soup_disk_open": (c_int32, [ctypes.POINTER(ctypes.c_char_p), c_int32, c_size_t, c_int32, c_int32, c_int32,
                                 c_int32, ctypes.POINTER(c_void_p)]),
    "soup_disk_close": (c_int32, [c_void_p]),
    "soup_disk_schedule": (c_int32, [c_void_p, ctypes.POINTER(c_int32), c_int32]),
    "soup_disk_acquire": (c_int32, [c_void_p, c_int32, c_int32, ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p)]),
    "soup_disk_release": (c_int32, [c_void_p, c_int32]),
    "soup_disk_stats": (c_int32, [c_void_p, ctypes.POINTER(DiskStats)]),
    "soup_stream_wait": (c_int32, [c_void_p, c_int32, c_void_p, ctypes.POINTER(c_void_p)]),
    "soup_stream_wait_host": (c_int32, [c_void_p, c_int32, c_int32]),
    "soup_stream_release": (c_int32, [c_void_p, c_int32, c_void_p]),
    "soup_stream_stats": (c_int32, [c_void_p, ctypes.POINTER(StreamStats)]),
    "soup_stream_stats_reset": (c_int32, [c_void_p]),
    "soup_stream_copy_stream": (c_void_p, [c_void_p]),
    "soup_stream_debug_timing_events": (c_int64, [c_void_p]),
    "soup_static_device_bytes": (c_size_t, []),
    "soup_gather_rows": (c_int32, [c_void_p, c_int64, c_void_p, c_int64, c_void_p, c_void_p]),
    "soup_sum_rows_f32": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "soup_attention_fwd": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_int32, c_int32, c_int32, c_int64,
                                     c_void_p, c_void_p, c_void_p, c_void_p]),
    "soup_attention_bwd": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_int32, c_int32, c_int32, c_int64,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "soup_debug_gemm_bounded_wait": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64,
                                               c_int32, c_void_p]),
    "soup_stream_debug_fail_next_copy": (c_int32, [c_void_p]),
    "soup_stream_debug_gate_next_copy": (c_int32, [c_void_p, c_void_p]),
    "soup_layer_blob_bytes": (c_size_t, [ctypes.POINTER(LayerCfg), c_int32]),
    "soup_layer_blob_views": (c_int32, [ctypes.POINTER(LayerCfg), c_int32, c_void_p, ctypes.POINTER(LayerWeights)]),
    "soup_embed": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_int64, c_void_p, c_void_p]),
    "soup_head_workspace": (c_size_t, [c_int64, c_int64, c_int64, c_int64, c_int32]),
    "soup_head_fwd_bwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_int64, c_int64,
                                    c_float, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "soup_ce_loss": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
    "soup_dpo_loss": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_float, c_void_p, c_void_p,
                                c_void_p, c_void_p]),
    "soup_simpo_loss": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_float, c_float, c_void_p, c_void_p,
                                  c_void_p, c_void_p]),
    "soup_orpo_loss": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_float, c_void_p, c_void_p, c_void_p,
                                 c_void_p]),
    "soup_adamw_step": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_float, c_float,
                                  c_float, c_float, c_float, c_float, c_int64, c_int32, c_void_p, c_void_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m layer_streamed_qlora_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn, st):
    if st != 0:
        msg = lib().soup_last_error()
        raise SoupError(fn, st, msg.decode() if msg else "")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def device_error() -> int:
    v = c_int32(0)
    _check("soup_device_error", lib().soup_device_error(ctypes.byref(v)))
    return v.value


def launch_count() -> int:
    return int(lib().soup_launch_count())


def profile_enable(class_mask: int):
    """class_mask bit c enables timing of kernel class c (PROFILE_CLASSES order); 0 disables."""
    _check("soup_profile_enable", lib().soup_profile_enable(int(class_mask)))


def profile_read() -> dict:
    arr = (GemmProfile * len(PROFILE_CLASSES))()
    _check("soup_profile_read", lib().soup_profile_read(arr, len(PROFILE_CLASSES)))
    return {name: {k: getattr(arr[i], k) for k, _ in GemmProfile._fields_} for i, name in enumerate(PROFILE_CLASSES)}


def soup_debug_gemm_bounded_wait(A, B, C, wait_limit_cycles=0, skip_producer_arrivals=False, stream=None):
    """C = A B^T (A [M, K], B [N, K] bf16; C [M, N] fp32) on the one-CTA GEMM
    engine with a caller-set mbarrier wait limit; with skip_producer_arrivals
    the producer never arrives and the kernel's wait runs out (device error 1)."""
    M, K = A.shape
    N = B.shape[0]
    _check("soup_debug_gemm_bounded_wait", lib().soup_debug_gemm_bounded_wait(
        _p(A), _p(B), M, N, K, _p(C), int(wait_limit_cycles), 1 if skip_producer_arrivals else 0, _stream(stream)))


def soup_attention_fwd(qkv, batch, seq, n_q, n_kv, out, out16, lse, prefix_share=1, prefix_len=0, stream=None):
    """Causal GQA attention forward on the q|k|v rows (fp16 [T, ld]); groups of
    prefix_share sequences may share a prefix of prefix_len tokens stored once."""
    _check("soup_attention_fwd", lib().soup_attention_fwd(_p(qkv), qkv.shape[1], batch, seq, n_q, n_kv,
                                                          prefix_share, prefix_len, _p(out), _p(out16), _p(lse),
                                                          _stream(stream)))


def soup_attention_bwd(qkv, batch, seq, n_q, n_kv, out16, dout, lse, D, dqkv, dqkv32=None, prefix_share=1,
                       prefix_len=0, stream=None):
    """Backward of soup_attention_fwd: dq|dk|dv into dqkv (bf16, qkv's layout)."""
    _check("soup_attention_bwd", lib().soup_attention_bwd(_p(qkv), qkv.shape[1], batch, seq, n_q, n_kv,
                                                          prefix_share, prefix_len, _p(out16), _p(dout), _p(lse),
                                                          _p(D), _p(dqkv), _p(dqkv32), _stream(stream)))


def soup_gather_rows(src, idx, dst, stream=None):
    """dst[i] = src[idx[i]] row by row (src, dst: device tensors of equal row size)."""
    n = idx.numel()
    rb = dst.numel() * dst.element_size() // max(1, n)
    _check("soup_gather_rows", lib().soup_gather_rows(_p(src), rb, _p(idx), n, _p(dst), _stream(stream)))


def soup_sum_rows_f32(src, src_idx, start, dst, stream=None):
    """dst[d] = sum of src rows src_idx[start[d]:start[d+1]] (fp32 [*, H])."""
    H = dst.shape[-1]
    n_dst = dst.numel() // H
    _check("soup_sum_rows_f32", lib().soup_sum_rows_f32(_p(src), H, _p(src_idx), _p(start), n_dst, _p(dst),
                                                        _stream(stream)))


def static_device_bytes() -> int:
    """Device bytes the library holds in module-static arrays on every device
    that loads it (held until process exit, outside any allocator)."""
    return int(lib().soup_static_device_bytes())


# ---------------------------------------------------------------- NF4
def soup_nf4_quantize(W, codes, absmax, flag, stream=None):
    out_f, in_f = W.shape
    _check("soup_nf4_quantize", lib().soup_nf4_quantize(_p(W), out_f, in_f, _p(codes), _p(absmax), _p(flag),
                                                        _stream(stream)))


def soup_nf4_dequant(codes, absmax, out_f, in_f, W_bf16, stream=None):
    _check("soup_nf4_dequant", lib().soup_nf4_dequant(_p(codes), _p(absmax), out_f, in_f, _p(W_bf16),
                                                      _stream(stream)))


# ---------------------------------------------------------------- weights
def weight_nf4(codes, absmax, out_f, in_f) -> SoupWeight:
    return SoupWeight(SOUP_WEIGHT_NF4, out_f, in_f, codes.data_ptr(), absmax.data_ptr(), None)


def weight_bf16(w) -> SoupWeight:
    return SoupWeight(SOUP_WEIGHT_BF16, w.shape[0], w.shape[1], None, None, w.data_ptr())


# ---------------------------------------------------------------- LoRA linear
def soup_lora_linear_fwd(W: SoupWeight, A, B, r, scale, x, T, y, u_save, stream=None):
    _check("soup_lora_linear_fwd", lib().soup_lora_linear_fwd(ctypes.byref(W), _p(A), _p(B), r, scale, _p(x), T,
                                                              _p(y), _p(u_save), _stream(stream)))


def soup_lora_linear_bwd_workspace(T, r, out_f) -> int:
    return int(lib().soup_lora_linear_bwd_workspace(T, r, out_f))


def soup_lora_linear_bwd(W: SoupWeight, A, B, r, scale, x, u_save, dy, T, dx, dA, dB, workspace, stream=None):
    _check("soup_lora_linear_bwd", lib().soup_lora_linear_bwd(
        ctypes.byref(W), _p(A), _p(B), r, scale, _p(x), _p(u_save), _p(dy), T, _p(dx), _p(dA), _p(dB),
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_lora_linear_bwd_noalloc_max_scratch() -> int:
    return int(lib().soup_lora_linear_bwd_noalloc_max_scratch())


def soup_lora_linear_bwd_noalloc(W: SoupWeight, A, B, r, scale, x, u_save, dy, T, dx, dA, dB, stream=None):
    """soup_lora_linear_bwd without a workspace (static scratch; see soup.h)."""
    _check("soup_lora_linear_bwd_noalloc", lib().soup_lora_linear_bwd_noalloc(
        ctypes.byref(W), _p(A), _p(B), r, scale, _p(x), _p(u_save), _p(dy), T, _p(dx), _p(dA), _p(dB),
        _stream(stream)))


# ---------------------------------------------------------------- decoder layer
def layer_cfg(shape) -> LayerCfg:
    return LayerCfg(shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, shape.intermediate,
                    shape.rank, float(shape.alpha), float(shape.eps), float(shape.theta))


def layer_lora(t: dict) -> LayerLora:
    return LayerLora(*[t[n].data_ptr() for n in ("A_qkv", "B_qkv", "A_o", "B_o", "A_gu", "B_gu", "A_down",
                                                 "B_down")])


def layer_grads(t: dict) -> LayerGrads:
    return LayerGrads(*[t[n].data_ptr() for n in ("dA_qkv", "dB_qkv", "dA_o", "dB_o", "dA_gu", "dB_gu",
                                                  "dA_down", "dB_down")])


def soup_decoder_layer_workspace(cfg: LayerCfg, batch, seq) -> int:
    return int(lib().soup_decoder_layer_workspace(ctypes.byref(cfg), batch, seq))


def soup_decoder_layer_fwd(W: LayerWeights, lora, cfg: LayerCfg, h_in, batch, seq, h_out, adapters_on, workspace,
                           stream=None):
    lp = ctypes.byref(lora) if lora is not None else None
    _check("soup_decoder_layer_fwd", lib().soup_decoder_layer_fwd(
        ctypes.byref(W), lp, ctypes.byref(cfg), _p(h_in), batch, seq, _p(h_out), int(adapters_on), _p(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_decoder_layer_bwd(W: LayerWeights, lora, cfg: LayerCfg, h_in, dh_out, batch, seq, dh_in, grads,
                           adapters_on, workspace, stream=None):
    lp = ctypes.byref(lora) if lora is not None else None
    gp = ctypes.byref(grads) if grads is not None else None
    _check("soup_decoder_layer_bwd", lib().soup_decoder_layer_bwd(
        ctypes.byref(W), lp, ctypes.byref(cfg), _p(h_in), _p(dh_out), batch, seq, _p(dh_in), gp, int(adapters_on),
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_decoder_layer_keep_bytes(cfg: LayerCfg, batch, seq) -> int:
    return int(lib().soup_decoder_layer_keep_bytes(ctypes.byref(cfg), batch, seq))


def soup_decoder_layer_fwd_keep(W: LayerWeights, lora, cfg: LayerCfg, h_in, batch, seq, h_out, adapters_on, qkv_keep,
                                workspace, stream=None):
    lp = ctypes.byref(lora) if lora is not None else None
    _check("soup_decoder_layer_fwd_keep", lib().soup_decoder_layer_fwd_keep(
        ctypes.byref(W), lp, ctypes.byref(cfg), _p(h_in), batch, seq, _p(h_out), int(adapters_on), _p(qkv_keep),
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_decoder_layer_bwd_kept(W: LayerWeights, lora, cfg: LayerCfg, h_in, dh_out, batch, seq, dh_in, grads,
                                adapters_on, qkv_kept, workspace, stream=None):
    lp = ctypes.byref(lora) if lora is not None else None
    gp = ctypes.byref(grads) if grads is not None else None
    _check("soup_decoder_layer_bwd_kept", lib().soup_decoder_layer_bwd_kept(
        ctypes.byref(W), lp, ctypes.byref(cfg), _p(h_in), _p(dh_out), batch, seq, _p(dh_in), gp, int(adapters_on),
        _p(qkv_kept), _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_decoder_layer_saved_bytes(cfg: LayerCfg, batch, seq) -> int:
    return int(lib().soup_decoder_layer_saved_bytes(ctypes.byref(cfg), batch, seq))


def soup_decoder_layer_fwd_save(W: LayerWeights, lora, cfg: LayerCfg, h_in, batch, seq, h_out, adapters_on, saved,
                                workspace, stream=None):
    lp = ctypes.byref(lora) if lora is not None else None
    _check("soup_decoder_layer_fwd_save", lib().soup_decoder_layer_fwd_save(
        ctypes.byref(W), lp, ctypes.byref(cfg), _p(h_in), batch, seq, _p(h_out), int(adapters_on), _p(saved),
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_decoder_layer_bwd_saved(W: LayerWeights, lora, cfg: LayerCfg, h_in, dh_out, batch, seq, dh_in, grads,
                                 adapters_on, saved, workspace, stream=None):
    lp = ctypes.byref(lora) if lora is not None else None
    gp = ctypes.byref(grads) if grads is not None else None
    _check("soup_decoder_layer_bwd_saved", lib().soup_decoder_layer_bwd_saved(
        ctypes.byref(W), lp, ctypes.byref(cfg), _p(h_in), _p(dh_out), batch, seq, _p(dh_in), gp, int(adapters_on),
        _p(saved), _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


# ---------------------------------------------------------------- streaming
class Plan:
    """Owns a soup_plan (slot arena + copy stream)."""

    def __init__(self, host_layers, layer_bytes, n_buffers, vocab_bytes=0, host_embed=None, host_head=None,
                 device_cap_bytes=0, reserve_bytes=0, n_layers=None):
        """host_layers: pinned host blobs, one per layer, or None (then
        n_layers gives the count and every layer copy comes through
        prefetch_from, e.g. from a Disk reader)."""
        if host_layers is None:
            n = int(n_layers)
            arr = None
        else:
            n = len(host_layers)
            self._arr = (c_void_p * n)(*[t.data_ptr() for t in host_layers])
            arr = ctypes.cast(self._arr, ctypes.POINTER(c_void_p))
        self._keep = (host_layers, host_embed, host_head)
        d = StreamDesc(n, layer_bytes, arr, vocab_bytes,
                       host_embed.data_ptr() if host_embed is not None else None,
                       host_head.data_ptr() if host_head is not None else None, n_buffers, device_cap_bytes,
                       reserve_bytes)
        h = c_void_p()
        _check("soup_stream_plan", lib().soup_stream_plan(ctypes.byref(d), ctypes.byref(h)))
        self.h = h

    def free(self):
        if self.h:
            lib().soup_stream_plan_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass

    def prefetch(self, item):
        _check("soup_stream_prefetch", lib().soup_stream_prefetch(self.h, item))

    def prefetch_from(self, layer, host_ptr: int, copy_done_event=None):
        _check("soup_stream_prefetch_from", lib().soup_stream_prefetch_from(self.h, layer, c_void_p(host_ptr),
                                                                            c_void_p(copy_done_event)))

    def resident(self, item) -> bool:
        r = c_int32(0)
        _check("soup_stream_resident", lib().soup_stream_resident(self.h, item, ctypes.byref(r)))
        return bool(r.value)

    def wait(self, item, stream=None) -> int:
        p = c_void_p()
        _check("soup_stream_wait", lib().soup_stream_wait(self.h, item, _stream(stream), ctypes.byref(p)))
        return p.value

    def wait_host(self, item, timeout_ms):
        _check("soup_stream_wait_host", lib().soup_stream_wait_host(self.h, item, timeout_ms))

    def release(self, item, stream=None):
        _check("soup_stream_release", lib().soup_stream_release(self.h, item, _stream(stream)))

    def stats(self) -> dict:
        s = StreamStats()
        _check("soup_stream_stats", lib().soup_stream_stats(self.h, ctypes.byref(s)))
        return {k: getattr(s, k) for k, _ in StreamStats._fields_}

    def reset_stats(self):
        _check("soup_stream_stats_reset", lib().soup_stream_stats_reset(self.h))

    def copy_stream_handle(self) -> int:
        return lib().soup_stream_copy_stream(self.h)

    def timing_events(self) -> int:
        return int(lib().soup_stream_debug_timing_events(self.h))

    def debug_fail_next_copy(self):
        _check("soup_stream_debug_fail_next_copy", lib().soup_stream_debug_fail_next_copy(self.h))

    def debug_gate_next_copy(self, event_handle):
        _check("soup_stream_debug_gate_next_copy", lib().soup_stream_debug_gate_next_copy(self.h, c_void_p(event_handle)))


def soup_layer_blob_bytes(cfg: LayerCfg, kind) -> int:
    return int(lib().soup_layer_blob_bytes(ctypes.byref(cfg), kind))


def soup_layer_blob_views(cfg: LayerCfg, kind, base_ptr: int) -> LayerWeights:
    w = LayerWeights()
    _check("soup_layer_blob_views", lib().soup_layer_blob_views(ctypes.byref(cfg), kind, c_void_p(base_ptr),
                                                                ctypes.byref(w)))
    return w


# ---------------------------------------------------------------- embedding / head / losses
def soup_embed(E_ptr: int, V, H, ids, T, h, stream=None):
    _check("soup_embed", lib().soup_embed(c_void_p(E_ptr), V, H, _p(ids), T, _p(h), _stream(stream)))


def soup_head_workspace(V, H, batch, seq, chunk) -> int:
    return int(lib().soup_head_workspace(V, H, batch, seq, chunk))


def soup_head_fwd_bwd(h, w_final, E_ptr: int, V, H, ids, batch, seq, eps, chunk, coef, logp, dh, workspace,
                      stream=None):
    _check("soup_head_fwd_bwd", lib().soup_head_fwd_bwd(
        _p(h), _p(w_final), c_void_p(E_ptr), V, H, _p(ids), batch, seq, eps, chunk, _p(coef), _p(logp), _p(dh),
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def soup_ce_loss(logp, batch, seq, loss, coef, stream=None):
    _check("soup_ce_loss", lib().soup_ce_loss(_p(logp), batch, seq, _p(loss), _p(coef), _stream(stream)))


def soup_dpo_loss(logp_policy, logp_ref, pairs, seq, prompt_len, beta, loss, seq_sums, coef, stream=None):
    _check("soup_dpo_loss", lib().soup_dpo_loss(_p(logp_policy), _p(logp_ref), pairs, seq, prompt_len, beta,
                                                _p(loss), _p(seq_sums), _p(coef), _stream(stream)))


def soup_simpo_loss(logp, pairs, seq, prompt_len, beta, gamma, loss, seq_sums, coef, stream=None):
    _check("soup_simpo_loss", lib().soup_simpo_loss(_p(logp), pairs, seq, prompt_len, beta, gamma, _p(loss),
                                                    _p(seq_sums), _p(coef), _stream(stream)))


def soup_orpo_loss(logp, pairs, seq, prompt_len, lam, loss, seq_sums, coef, stream=None):
    _check("soup_orpo_loss", lib().soup_orpo_loss(_p(logp), pairs, seq, prompt_len, lam, _p(loss), _p(seq_sums),
                                                  _p(coef), _stream(stream)))


def soup_adamw_step(theta, theta_bf16, grad, m, v, lr, beta1, beta2, eps, weight_decay, grad_scale, t,
                    zero_grad=True, nonfinite=None, stream=None):
    """One AdamW step over flat fp32 buffers (theta, grad, m, v of equal
    length; theta_bf16 the bf16 working copy or None)."""
    n = theta.numel()
    for x in (grad, m, v) + (() if theta_bf16 is None else (theta_bf16,)):
        assert x.numel() == n and x.is_contiguous()
    _check("soup_adamw_step", lib().soup_adamw_step(_p(theta), _p(theta_bf16), _p(grad), _p(m), _p(v), n, lr, beta1,
                                                    beta2, eps, weight_decay, grad_scale, t, 1 if zero_grad else 0,
                                                    _p(nonfinite), _stream(stream)))


class Disk:
    """Owns a soup_disk reader: per-layer shard files read ahead into
    `read_ahead` staging buffers along a cyclic layer visit schedule."""

    def __init__(self, paths, layer_bytes, read_ahead=2, n_slots=2, io_threads=4, pinned=True, direct=True):
        self._paths = (ctypes.c_char_p * len(paths))(*[os.fsencode(p) for p in paths])
        flags = (SOUP_DISK_PINNED if pinned else 0) | (SOUP_DISK_DIRECT if direct else 0)
        h = c_void_p()
        _check("soup_disk_open", lib().soup_disk_open(self._paths, len(paths), layer_bytes, read_ahead, n_slots,
                                                      io_threads, flags, ctypes.byref(h)))
        self.h = h
        self.layer_bytes = layer_bytes

    def schedule(self, order):
        arr = (c_int32 * len(order))(*order)
        _check("soup_disk_schedule", lib().soup_disk_schedule(self.h, arr, len(order)))

    def acquire(self, layer, timeout_ms=60000):
        """Returns (host address, copy-done cudaEvent_t or None)."""
        host, ev = c_void_p(), c_void_p()
        _check("soup_disk_acquire", lib().soup_disk_acquire(self.h, layer, timeout_ms, ctypes.byref(host),
                                                            ctypes.byref(ev)))
        return host.value, ev.value

    def release(self, layer):
        _check("soup_disk_release", lib().soup_disk_release(self.h, layer))

    def stats(self) -> dict:
        s = DiskStats()
        _check("soup_disk_stats", lib().soup_disk_stats(self.h, ctypes.byref(s)))
        return {k: getattr(s, k) for k, _ in DiskStats._fields_}

    def close(self):
        if self.h:
            lib().soup_disk_close(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
