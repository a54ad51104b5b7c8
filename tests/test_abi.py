"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/flexq.h declares, and rejects bad arguments on the host before
any launch (no compute call is made here)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flexq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flexq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def fq():
    from quantized_opt_decode_b200 import build
    build.build()
    from quantized_opt_decode_b200 import flexq
    return flexq


def test_header_declares_the_pages_entry_points():
    names = declared_functions()
    for must in ("flexq_quantize", "flexq_dequantize", "flexq_layer_prefill",
                 "flexq_layer_decode", "flexq_kv_append", "flexq_generate"):
        assert must in names


def test_every_declared_symbol_is_exported(fq):
    lib = C.CDLL(fq._LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_functions()) == set(fq.EXPORTED)


def test_version_and_empty_error(fq):
    assert fq.flexq_version() == 102


def _status(fn, *args):
    return fn(*args)


def test_codec_rejects_ragged_length(fq):
    lib = fq._lib
    assert lib.flexq_quantize(None, 65, None, None, None, None) == 1
    assert "multiple of 64" in fq.flexq_last_error()
    assert lib.flexq_dequantize(None, None, None, 100, None, None) == 1


def test_codec_rejects_null_and_misaligned(fq):
    lib = fq._lib
    assert lib.flexq_quantize(None, 64, None, None, None, None) == 1
    assert lib.flexq_quantize(0x1001, 64, 0x2000, 0x3000, 0x4000, None) == 1
    assert "aligned" in fq.flexq_last_error()


def test_packed_weight_size(fq):
    assert fq.flexq_packed_weight_bytes(256, 128) == 2 * 2 * 4608
    assert fq.flexq_packed_weight_bytes(130, 64) == 2 * 1 * 4608
    assert fq.flexq_packed_weight_bytes(128, 65) == 0


def test_config_validation(fq):
    bad = [dict(h=100, heads=1), dict(h=256, heads=3), dict(h=256, heads=1),
           dict(h=256, heads=4, ffn=100), dict(h=256, heads=4, w_bits=8),
           dict(attn_topk_permille=1001), dict(attn_topk_permille=-1),
           dict(kv_bits=16, attn_topk_permille=100), dict(prefill_kv_cache=2)]
    for over in bad:
        kw = dict(h=256, heads=4, ffn=1024, w_bits=4, kv_bits=4, ln_eps=1e-5)
        kw.update(over)
        cfg = fq.flexq_config(**kw)
        assert fq._lib.flexq_kv_bytes(C.byref(cfg), 1, 8) == 0
        assert fq._lib.flexq_layer_workspace(C.byref(cfg), 4, 1) == 0


def test_kv_bytes_closed_forms(fq):
    """fp16: 2 (K and V) * 2 bytes * b * L * h; 4-bit: 0.5 byte per element
    plus 4 bytes of (min, scale) per 64 elements."""
    for bits in (16, 4):
        cfg = fq.flexq_config(h=7168, heads=56, ffn=28672, w_bits=4, kv_bits=bits, ln_eps=1e-5)
        b, L = 144, 544
        n = fq.flexq_kv_bytes(cfg, b, L)
        per_elem = 2.0 if bits == 16 else 0.5 + 4 / 64
        assert n == int(2 * per_elem * b * L * 7168)


def test_layer_rejects_bad_arguments(fq):
    cfg = fq.flexq_config(h=256, heads=4, ffn=1024, w_bits=4, kv_bits=4, ln_eps=1e-5)
    layer = fq.flexq_layer()
    kv = fq.flexq_kv(0x1000, 0x2000, 0x3000, 0x4000, 4, 40)
    st = fq._lib.flexq_layer_decode(C.byref(cfg), C.byref(layer), 0x1000, 0x2000, C.byref(kv), 4,
                                    3, None, 0, None)
    assert st == 1 and "NULL" in fq.flexq_last_error()
    st = fq._lib.flexq_layer_decode(C.byref(cfg), None, 0x1000, 0x2000, C.byref(kv), 4, 50, None,
                                    0, None)
    assert st == 1 and "pos" in fq.flexq_last_error()


def test_layer_rejects_short_workspace(fq):
    cfg = fq.flexq_config(h=256, heads=4, ffn=1024, w_bits=16, kv_bits=16, ln_eps=1e-5)
    ptrs = [0x10000 * (i + 1) for i in range(12)]
    layer = fq.flexq_layer(*ptrs)
    kv = fq.flexq_kv(0x100000, 0x200000, None, None, 4, 40)
    need = fq._lib.flexq_layer_workspace(C.byref(cfg), 4, 1)
    assert need > 0
    st = fq._lib.flexq_layer_decode(C.byref(cfg), C.byref(layer), 0x300000, 0x400000, C.byref(kv),
                                    4, 3, 0x500000, need - 1, None)
    assert st == 3


def test_generate_rejects_indivisible_gpu_batch(fq):
    cfg = fq.flexq_config(h=256, heads=4, ffn=1024, w_bits=16, kv_bits=16, ln_eps=1e-5)
    ptrs = [0x10000 * (i + 1) for i in range(12)]
    layer = (fq.flexq_layer * 1)(fq.flexq_layer(*ptrs))
    kv = (fq.flexq_kv * 1)(fq.flexq_kv(0x100000, 0x200000, None, None, 4, 40))
    m = fq.flexq_model(cfg, 1, 512, 40, layer, kv, 0x1000, 0x2000, 0x3000, 0x4000, 16)
    st = fq._lib.flexq_generate(C.byref(m), 0x5000, 4, 32, 8, 3, 0x6000, 0x7000, 1 << 30, None,
                                None)
    assert st == 1 and "gpu_batch" in fq.flexq_last_error()
    m.embed_bits = 8
    st = fq._lib.flexq_generate(C.byref(m), 0x5000, 4, 32, 8, 4, 0x6000, 0x7000, 1 << 30, None,
                                None)
    assert st == 1 and "embed_bits" in fq.flexq_last_error()
    m.embed_bits = 16
    # s + n - 1 = 41 positions exceed max_pos = 40
    st = fq._lib.flexq_generate(C.byref(m), 0x5000, 4, 32, 10, 4, 0x6000, 0x7000, 1 << 30, None,
                                None)
    assert st == 1 and "max_pos" in fq.flexq_last_error()


def test_package_builds_from_scratch_and_binding_fails_loudly(tmp_path):
    """Without libflexq.so the package still imports (so its build module can
    compile the library on a fresh checkout), and the binding refuses to load:
    there is no fallback path."""
    import shutil
    import subprocess
    import sys
    src = os.path.join(ROOT, "quantized_opt_decode_b200")
    dst = tmp_path / "quantized_opt_decode_b200"
    dst.mkdir()
    for f in os.listdir(src):
        if f.endswith(".py"):
            shutil.copy(os.path.join(src, f), dst / f)
    code = ("import quantized_opt_decode_b200 as q, quantized_opt_decode_b200.build as b\n"
            "try:\n    q.flexq\nexcept ImportError as e:\n    print('refused:', e)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True,
                       env=dict(os.environ, PYTHONPATH=str(tmp_path)))
    assert r.returncode == 0, r.stderr
    assert "refused:" in r.stdout and "libflexq.so" in r.stdout


def test_prefill_cache_rejects_bad_arguments(fq):
    cfg = fq.flexq_config(h=256, heads=4, ffn=1024, w_bits=4, kv_bits=4, ln_eps=1e-5)
    kv = fq.flexq_kv(0x1000, 0x2000, 0x3000, 0x4000, 4, 40)
    st = fq._lib.flexq_attention_prefill_cache(C.byref(cfg), C.byref(kv), 0x1000, 256, 4, 36, 8, 0x2000, 256,
                                               None)
    assert st == 1 and "exceed" in fq.flexq_last_error()
    st = fq._lib.flexq_attention_prefill_cache(C.byref(cfg), C.byref(kv), 0x1000, 256, 4, 16, 4, 0x2000, 256,
                                               None)
    assert st == 1 and "pos0" in fq.flexq_last_error()


def test_linear_rejects_bad_arguments(fq):
    lib = fq._lib
    A = 0x100000  # 16-byte aligned placeholders; nothing is launched on a rejection
    st = lib.flexq_linear(A, 64, A, 8, 4, 128, 64, None, None, 0, 0, A, 128, None, 0, 0, None)
    assert st == 1 and "w_bits" in fq.flexq_last_error()
    st = lib.flexq_linear(A, 96, A, 4, 4, 128, 96, None, None, 0, 0, A, 128, None, 0, 0, None)
    assert st == 1 and "multiple of 64" in fq.flexq_last_error()
    st = lib.flexq_linear(A + 2, 64, A, 4, 4, 128, 64, None, None, 0, 0, A, 128, None, 0, 0, None)
    assert st == 1 and "alignment" in fq.flexq_last_error()
    st = lib.flexq_linear(A, 64, A, 4, 4, 128, 64, None, None, 0, 1, A, 128, None, 0, 0, None)
    assert st == 1 and "bias" in fq.flexq_last_error()
    st = lib.flexq_linear(A, 64, A, 4, 4, 128, 64, A, None, 0, 8 | 1, A, 128, None, 0, 0, None)
    assert st == 1 and "fp32 output" in fq.flexq_last_error()
    st = lib.flexq_linear(A, 64, A, 4, 4, 128, 64, None, None, 0, 0, A, 128, None, 0, 2, None)
    assert st == 1 and "force_splits" in fq.flexq_last_error()


def test_kv_append_and_attention_reject_bad_arguments(fq):
    cfg = fq.flexq_config(h=256, heads=4, ffn=1024, w_bits=4, kv_bits=4, ln_eps=1e-5)
    kv = fq.flexq_kv(0x1000, 0x2000, 0x3000, 0x4000, 4, 40)
    lib, A = fq._lib, 0x100000
    st = lib.flexq_kv_append(C.byref(cfg), C.byref(kv), A, A, 768, 4, 38, 3, None)
    assert st == 1 and "outside max_len" in fq.flexq_last_error()
    st = lib.flexq_attention_decode(C.byref(cfg), C.byref(kv), A, 768, 4, 41, A, 256, None)
    assert st == 1 and "max_len" in fq.flexq_last_error()
    st = lib.flexq_attention_decode(C.byref(cfg), C.byref(kv), A, 770, 4, 16, A, 256, None)
    assert st == 1 and "strides" in fq.flexq_last_error()
    long_kv = fq.flexq_kv(0x1000, 0x2000, 0x3000, 0x4000, 4, 20000)
    st = lib.flexq_attention_decode(C.byref(cfg), C.byref(long_kv), A, 768, 4, 16385, A, 256, None)
    assert st == 1 and "16384" in fq.flexq_last_error()
    st = lib.flexq_attention_decode_topk(C.byref(cfg), C.byref(kv), A, 768, 4, 16, 17, A, 256, None, None)
    assert st == 1 and "k must" in fq.flexq_last_error()
    cfg16 = fq.flexq_config(h=256, heads=4, ffn=1024, w_bits=4, kv_bits=16, ln_eps=1e-5)
    kv16 = fq.flexq_kv(0x1000, 0x2000, None, None, 4, 40)
    st = lib.flexq_attention_decode_topk(C.byref(cfg16), C.byref(kv16), A, 768, 4, 16, 2, A, 256, None, None)
    assert st == 1 and "4-bit" in fq.flexq_last_error()
