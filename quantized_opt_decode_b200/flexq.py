"""ctypes binding of libflexq.so (include/flexq.h).

Argument marshalling only: every function here has the C entry point's name,
accepts torch tensors (their data_ptr() is passed) or plain integers for
device pointers, raises FlexqError on a non-zero status and returns what the C
function returns otherwise.  Nothing is computed in Python.  The binding
refuses to load without the compiled library: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libflexq.so")

FLEXQ_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID", 2: "CUDA", 3: "WORKSPACE", 4: "TIMEOUT",
                5: "UNSUPPORTED", 6: "DEVICE"}
EPI_BIAS, EPI_GELU, EPI_RESIDUAL, EPI_F32_OUT = 1, 2, 4, 8
KERNEL_KINDS = ("layernorm", "qkv", "kv_append", "attn_prefill", "attn_decode", "out_proj", "fc1",
                "fc2", "embed", "lm_head", "argmax")


class FlexqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"flexq status {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libflexq.so not found at {_LIB_PATH}; build it with "
            "`python -m quantized_opt_decode_b200.build` (nvcc, sm_100a)")
    return C.CDLL(_LIB_PATH)


_lib = _load()
VP = C.c_void_p


class flexq_config(C.Structure):
    _fields_ = [("h", C.c_int), ("heads", C.c_int), ("ffn", C.c_int), ("w_bits", C.c_int),
                ("kv_bits", C.c_int), ("ln_eps", C.c_float), ("attn_topk_permille", C.c_int),
                ("prefill_kv_cache", C.c_int)]


class flexq_layer(C.Structure):
    _fields_ = [(n, VP) for n in ("w_qkv", "w_o", "w_fc1", "w_fc2", "b_qkv", "b_o", "b_fc1",
                                  "b_fc2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")]


class flexq_kv(C.Structure):
    _fields_ = [("k", VP), ("v", VP), ("k_meta", VP), ("v_meta", VP), ("b", C.c_int),
                ("max_len", C.c_int)]


class flexq_model(C.Structure):
    _fields_ = [("cfg", flexq_config), ("layers", C.c_int), ("vocab", C.c_int),
                ("max_pos", C.c_int), ("layer", C.POINTER(flexq_layer)),
                ("kv", C.POINTER(flexq_kv)), ("embed", VP), ("pos_embed", VP), ("lnf_g", VP),
                ("lnf_b", VP), ("embed_bits", C.c_int)]


class flexq_timing(C.Structure):
    _fields_ = [("prefill_ms", C.c_float), ("decode_ms", C.c_float)]


class flexq_hw(C.Structure):
    _fields_ = [("h2d_gbps", C.c_double), ("hbm_gbps", C.c_double), ("tensor_tflops", C.c_double),
                ("device_bytes", C.c_double)]


class flexq_offload_choice(C.Structure):
    _fields_ = [("gpu_batch", C.c_int), ("num_batches", C.c_int), ("decode_tokens_per_s", C.c_double),
                ("column_io_s", C.c_double), ("column_compute_s", C.c_double), ("device_bytes", C.c_double)]


_CFG = C.POINTER(flexq_config)
_SIGS = {
    "flexq_last_error": ([], C.c_char_p),
    "flexq_version": ([], C.c_int),
    "flexq_device_status": ([VP], C.c_int),
    "flexq_set_wait_limit_ns": ([C.c_uint64], C.c_int),
    "flexq_set_launch_overlap": ([C.c_int], C.c_int),
    "flexq_synth_normal_f16": ([VP, C.c_size_t, C.c_uint64, C.c_uint64, C.c_size_t, C.c_float,
                                C.c_float, VP], C.c_int),
    "flexq_synth_tokens": ([VP, C.c_size_t, C.c_uint64, C.c_uint64, C.c_size_t, C.c_int32, VP],
                           C.c_int),
    "flexq_quantize": ([VP, C.c_size_t, VP, VP, VP, VP], C.c_int),
    "flexq_dequantize": ([VP, VP, VP, C.c_size_t, VP, VP], C.c_int),
    "flexq_packed_weight_bytes": ([C.c_int, C.c_int], C.c_size_t),
    "flexq_pack_weight_q4": ([VP, VP, VP, C.c_int, C.c_int, VP, VP], C.c_int),
    "flexq_quantize_weight_q4": ([VP, C.c_int, C.c_int, VP, VP], C.c_int),
    "flexq_linear_workspace": ([C.c_int, C.c_int, C.c_int, C.c_int, C.c_int], C.c_size_t),
    "flexq_linear": ([VP, C.c_int, VP, C.c_int, C.c_int, C.c_int, C.c_int, VP, VP, C.c_int,
                      C.c_int, VP, C.c_int, VP, C.c_size_t, C.c_int, VP], C.c_int),
    "flexq_linear_static_scratch": ([VP, C.c_int, VP, C.c_int, C.c_int, C.c_int, C.c_int, VP, VP,
                                     C.c_int, C.c_int, VP, C.c_int, C.c_int, VP], C.c_int),
    "flexq_layernorm": ([VP, C.c_int, VP, VP, VP, C.c_int, C.c_int, C.c_int, C.c_float, VP],
                        C.c_int),
    "flexq_kv_bytes": ([_CFG, C.c_int, C.c_int], C.c_size_t),
    "flexq_kv_append": ([_CFG, C.POINTER(flexq_kv), VP, VP, C.c_int, C.c_int, C.c_int, C.c_int,
                         VP], C.c_int),
    "flexq_attention_decode": ([_CFG, C.POINTER(flexq_kv), VP, C.c_int, C.c_int, C.c_int, VP,
                                C.c_int, VP], C.c_int),
    "flexq_attention_decode_topk": ([_CFG, C.POINTER(flexq_kv), VP, C.c_int, C.c_int, C.c_int, C.c_int,
                                     VP, C.c_int, VP, VP], C.c_int),
    "flexq_attention_prefill": ([_CFG, VP, C.c_int, C.c_int, C.c_int, VP, C.c_int, VP], C.c_int),
    "flexq_attention_prefill_cache": ([_CFG, C.POINTER(flexq_kv), VP, C.c_int, C.c_int, C.c_int, C.c_int, VP,
                                       C.c_int, VP], C.c_int),
    "flexq_layer_workspace": ([_CFG, C.c_int, C.c_int], C.c_size_t),
    "flexq_layer_prefill": ([_CFG, C.POINTER(flexq_layer), VP, VP, C.POINTER(flexq_kv), C.c_int,
                             C.c_int, VP, C.c_size_t, VP], C.c_int),
    "flexq_layer_decode": ([_CFG, C.POINTER(flexq_layer), VP, VP, C.POINTER(flexq_kv), C.c_int,
                            C.c_int, VP, C.c_size_t, VP], C.c_int),
    "flexq_generate_workspace": ([C.POINTER(flexq_model), C.c_int, C.c_int, C.c_int],
                                 C.c_size_t),
    "flexq_generate": ([C.POINTER(flexq_model), VP, C.c_int, C.c_int, C.c_int, C.c_int, VP, VP,
                        C.c_size_t, C.POINTER(flexq_timing), VP], C.c_int),
    "flexq_generate_prefill": ([C.POINTER(flexq_model), VP, C.c_int, C.c_int, C.c_int, C.c_int, VP,
                                VP, C.c_size_t, VP], C.c_int),
    "flexq_generate_decode": ([C.POINTER(flexq_model), C.c_int, C.c_int, C.c_int, C.c_int, VP, VP,
                               C.c_size_t, VP], C.c_int),
    "flexq_offload_slot_bytes": ([_CFG], C.c_size_t),
    "flexq_generate_offload": ([C.POINTER(flexq_model), VP, C.c_size_t, VP, VP, C.c_int, C.c_int, C.c_int,
                                C.c_int, VP, VP, C.c_size_t, C.POINTER(flexq_timing), VP], C.c_int),
    "flexq_offload_plan": ([C.POINTER(flexq_model), C.c_int, C.c_int, C.POINTER(flexq_hw), C.c_int,
                            C.POINTER(flexq_offload_choice)], C.c_int),
    "flexq_launch_count": ([], C.c_uint64),
    "flexq_profile_start": ([], C.c_int),
    "flexq_profile_stop": ([VP, C.POINTER(C.c_float), C.POINTER(C.c_int)], C.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTED = tuple(_SIGS)


def _p(x):
    """Device pointer of a tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _s(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != FLEXQ_OK:
        raise FlexqError(status, _lib.flexq_last_error().decode())


def flexq_last_error() -> str:
    return _lib.flexq_last_error().decode()


def flexq_version() -> int:
    return _lib.flexq_version()


def flexq_device_status(stream=None):
    _check(_lib.flexq_device_status(_s(stream)))


def flexq_set_wait_limit_ns(ns: int):
    _check(_lib.flexq_set_wait_limit_ns(ns))


def flexq_set_launch_overlap(on: bool) -> bool:
    return bool(_lib.flexq_set_launch_overlap(1 if on else 0))


def flexq_synth_normal_f16(out, n, seed, tensor_id, start=0, sigma=0.02, mean=0.0, stream=None):
    _check(_lib.flexq_synth_normal_f16(_p(out), n, seed, tensor_id, start, sigma, mean, _s(stream)))


def flexq_synth_tokens(out, n, seed, tensor_id, vocab, start=0, stream=None):
    _check(_lib.flexq_synth_tokens(_p(out), n, seed, tensor_id, start, vocab, _s(stream)))


def flexq_quantize(x, n, codes, mn, sc, stream=None):
    _check(_lib.flexq_quantize(_p(x), n, _p(codes), _p(mn), _p(sc), _s(stream)))


def flexq_dequantize(codes, mn, sc, n, out, stream=None):
    _check(_lib.flexq_dequantize(_p(codes), _p(mn), _p(sc), n, _p(out), _s(stream)))


def flexq_packed_weight_bytes(n_out, k_in) -> int:
    return _lib.flexq_packed_weight_bytes(n_out, k_in)


def flexq_pack_weight_q4(codes, mn, sc, n_out, k_in, packed, stream=None):
    _check(_lib.flexq_pack_weight_q4(_p(codes), _p(mn), _p(sc), n_out, k_in, _p(packed),
                                     _s(stream)))


def flexq_quantize_weight_q4(w, n_out, k_in, packed, stream=None):
    _check(_lib.flexq_quantize_weight_q4(_p(w), n_out, k_in, _p(packed), _s(stream)))


def flexq_linear_workspace(m, n, k, w_bits, force_splits=0) -> int:
    return _lib.flexq_linear_workspace(m, n, k, w_bits, force_splits)


def flexq_linear(x, ldx, w, w_bits, m, n, k, bias, residual, ld_res, epilogue, y, ldy,
                 ws=None, ws_bytes=0, force_splits=0, stream=None):
    _check(_lib.flexq_linear(_p(x), ldx, _p(w), w_bits, m, n, k, _p(bias), _p(residual), ld_res,
                             epilogue, _p(y), ldy, _p(ws), ws_bytes, force_splits, _s(stream)))


def flexq_linear_static_scratch(x, ldx, w, w_bits, m, n, k, bias, residual, ld_res, epilogue, y,
                                ldy, force_splits=0, stream=None):
    _check(_lib.flexq_linear_static_scratch(_p(x), ldx, _p(w), w_bits, m, n, k, _p(bias),
                                            _p(residual), ld_res, epilogue, _p(y), ldy,
                                            force_splits, _s(stream)))


def flexq_layernorm(x, ldx, gamma, beta, y, ldy, rows, h, eps=1e-5, stream=None):
    _check(_lib.flexq_layernorm(_p(x), ldx, _p(gamma), _p(beta), _p(y), ldy, rows, h, eps,
                                _s(stream)))


def flexq_kv_bytes(cfg: flexq_config, b, max_len) -> int:
    return _lib.flexq_kv_bytes(C.byref(cfg), b, max_len)


def flexq_kv_append(cfg, kv, k, v, ld, b, pos0, ntok, stream=None):
    _check(_lib.flexq_kv_append(C.byref(cfg), C.byref(kv), _p(k), _p(v), ld, b, pos0, ntok,
                                _s(stream)))


def flexq_attention_decode(cfg, kv, q, ldq, b, length, out, ldo, stream=None):
    _check(_lib.flexq_attention_decode(C.byref(cfg), C.byref(kv), _p(q), ldq, b, length, _p(out),
                                       ldo, _s(stream)))


def flexq_attention_decode_topk(cfg, kv, q, ldq, b, length, k, out, ldo, idx=None, stream=None):
    _check(_lib.flexq_attention_decode_topk(C.byref(cfg), C.byref(kv), _p(q), ldq, b, length, k,
                                            _p(out), ldo, _p(idx), _s(stream)))


def flexq_attention_prefill(cfg, qkv, ldqkv, b, s, out, ldo, stream=None):
    _check(_lib.flexq_attention_prefill(C.byref(cfg), _p(qkv), ldqkv, b, s, _p(out), ldo,
                                        _s(stream)))


def flexq_attention_prefill_cache(cfg, kv, q, ldq, b, s, pos0, out, ldo, stream=None):
    _check(_lib.flexq_attention_prefill_cache(C.byref(cfg), C.byref(kv), _p(q), ldq, b, s, pos0, _p(out),
                                              ldo, _s(stream)))


def flexq_layer_workspace(cfg, rows, mode) -> int:
    return _lib.flexq_layer_workspace(C.byref(cfg), rows, mode)


def flexq_layer_prefill(cfg, layer, x, y, kv, b, s, ws, ws_bytes, stream=None):
    _check(_lib.flexq_layer_prefill(C.byref(cfg), C.byref(layer), _p(x), _p(y), C.byref(kv), b, s,
                                    _p(ws), ws_bytes, _s(stream)))


def flexq_layer_decode(cfg, layer, t, y, kv, b, pos, ws, ws_bytes, stream=None):
    _check(_lib.flexq_layer_decode(C.byref(cfg), C.byref(layer), _p(t), _p(y), C.byref(kv), b, pos,
                                   _p(ws), ws_bytes, _s(stream)))


def flexq_generate_workspace(model, b, s, gpu_batch) -> int:
    return _lib.flexq_generate_workspace(C.byref(model), b, s, gpu_batch)


def flexq_generate(model, prompt, b, s, n, gpu_batch, out, ws, ws_bytes, timing=None,
                   stream=None):
    _check(_lib.flexq_generate(C.byref(model), _p(prompt), b, s, n, gpu_batch, _p(out), _p(ws),
                               ws_bytes, C.byref(timing) if timing is not None else None,
                               _s(stream)))


def flexq_generate_prefill(model, prompt, b, s, n, gpu_batch, out, ws, ws_bytes, stream=None):
    _check(_lib.flexq_generate_prefill(C.byref(model), _p(prompt), b, s, n, gpu_batch, _p(out),
                                       _p(ws), ws_bytes, _s(stream)))


def flexq_generate_decode(model, b, s, n, gpu_batch, out, ws, ws_bytes, stream=None):
    _check(_lib.flexq_generate_decode(C.byref(model), b, s, n, gpu_batch, _p(out), _p(ws),
                                      ws_bytes, _s(stream)))


def flexq_offload_slot_bytes(cfg) -> int:
    return _lib.flexq_offload_slot_bytes(C.byref(cfg))


def flexq_generate_offload(model, slots, slots_bytes, copy_stream, prompt, b, s, n, gpu_batch, out, ws,
                           ws_bytes, timing=None, stream=None):
    _check(_lib.flexq_generate_offload(C.byref(model), _p(slots), slots_bytes, _s(copy_stream), _p(prompt), b,
                                       s, n, gpu_batch, _p(out), _p(ws), ws_bytes,
                                       C.byref(timing) if timing is not None else None, _s(stream)))


def flexq_offload_plan(model, s, n, hw, max_block):
    choice = flexq_offload_choice()
    _check(_lib.flexq_offload_plan(C.byref(model), s, n, C.byref(hw), max_block, C.byref(choice)))
    return choice


def flexq_launch_count() -> int:
    return _lib.flexq_launch_count()


def flexq_profile_start():
    _check(_lib.flexq_profile_start())


def flexq_profile_stop(stream=None):
    """-> {kind: (total_ms, calls)}"""
    ms = (C.c_float * len(KERNEL_KINDS))()
    calls = (C.c_int * len(KERNEL_KINDS))()
    _check(_lib.flexq_profile_stop(_s(stream), ms, calls))
    return {k: (ms[i], calls[i]) for i, k in enumerate(KERNEL_KINDS)}
