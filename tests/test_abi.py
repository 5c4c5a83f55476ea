"""C-ABI boundary checks that need no GPU: the library builds and loads,
exports every symbol the headers declare, and its host-side arithmetic and
argument checks behave (no kernel is launched by any call here)."""
import ctypes
import os
import math

import pytest

import oracle as O
from long_context_prefill_tcgen05_b200 import build, dash, inputs


@pytest.fixture(scope="module")
def L():
    build.build()
    return dash.lib()


def test_every_declared_symbol_is_exported(L):
    names = dash.declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, text in dash.STATUS.items():
        assert L.dash_status_string(code).decode() == text


@pytest.mark.parametrize("T", [0, 1, 7, 100, 512, 32768, 131072])
@pytest.mark.parametrize("keep", [0.0, 0.1, 0.333, 0.4, 0.5, 0.7, 1.0])
@pytest.mark.parametrize("nf,nl", [(0, 0), (64, 32), (3, 0), (0, 5), (200, 200)])
def test_topk_count_matches_oracle(L, T, keep, nf, nl):
    assert dash.topk_count(T, keep, nf, nl) == (O.topk_count(T, keep, nf, nl) if T > 0 else 0)


FAKE = 1 << 20  # an aligned non-null address; the calls below fail before using it


def _dims(**kw):
    d = inputs.TINY
    base = dict(n_layers=d.n_layers, d_model=d.d_model, n_heads=d.n_heads, n_kv_heads=d.n_kv_heads,
                head_dim=d.head_dim, ffn_dim=d.ffn_dim, rms_eps=d.rms_eps, rope_theta=d.rope_theta)
    base.update(kw)
    return dash.Dims(**base)


def _fake_layers(n):
    arr = (dash.LayerWeights * n)()
    for i in range(n):
        arr[i] = dash.LayerWeights(*([FAKE] * 7))
    return arr


def test_argument_errors_are_caught_on_the_host(L):
    dims = _dims()
    cfg = dash.make_config(halt_layer=2, mode="prune", keep=0.5)
    layers = _fake_layers(4)
    K = ctypes.c_int64(0)
    call = lambda d, lay, H, T, c, ws=None, wsb=0: L.dash_prefill(
        ctypes.byref(d), lay, H, T, ctypes.byref(c), None, ctypes.byref(K), None, ws, wsb, None)
    assert call(dims, layers, None, 512, cfg) == 1                       # null H
    assert call(_dims(head_dim=96), layers, FAKE, 512, cfg) == 2         # unsupported head_dim
    assert call(_dims(n_heads=3), layers, FAKE, 512, cfg) == 2           # hq % hkv != 0
    assert call(_dims(d_model=200), layers, FAKE, 512, cfg) == 2         # d % 128 != 0
    assert call(_dims(dtype=2), layers, FAKE, 512, cfg) == 2             # no such 16-bit format
    assert call(_dims(dtype=1), layers, FAKE, 512, cfg, None, 0) == 4    # fp16 accepted (then: no workspace)
    assert call(dims, layers, FAKE + 2, 512, cfg) == 1                   # misaligned H
    bad = dash.make_config(halt_layer=4, mode="prune")
    assert call(dims, layers, FAKE, 512, bad) == 1                       # halt layer out of range
    bad = dash.make_config(halt_layer=1, keep=1.5)
    assert call(dims, layers, FAKE, 512, bad) == 1                       # keep > 1
    bad = dash.make_config(halt_layer=1); bad.mode = 9
    assert call(dims, layers, FAKE, 512, bad) == 1                       # unknown mode
    bad = dash.make_config(halt_layer=1, monitor_layers=3)
    assert call(dims, layers, FAKE, 512, bad) == 1                       # window longer than layers 0..L_s
    holes = _fake_layers(4); holes[3] = dash.LayerWeights(*([FAKE] * 6 + [0]))
    assert call(dims, holes, FAKE, 512, cfg) == 1                        # a null weight
    assert call(dims, layers, FAKE, 512, cfg, None, 0) == 4              # no workspace
    need = L.dash_prefill_workspace_size(ctypes.byref(dims), 512, ctypes.byref(cfg))
    assert call(dims, layers, FAKE, 512, cfg, FAKE, need - 1) == 4       # workspace one byte short
    assert call(dims, layers, FAKE, 0, cfg) == 0 and K.value == 0        # empty input: nothing to do

    # select / score / compact shape and argument checks
    cnt = FAKE
    assert L.dash_select(FAKE, 10, 7, 0.5, 0.0, 0, 0, FAKE, None, cnt, None, 0, None) == 1
    assert L.dash_select(FAKE, 10, 0, -0.1, 0.0, 0, 0, FAKE, None, cnt, None, 0, None) == 1
    assert L.dash_select(FAKE, 10, 0, 0.5, 0.0, -1, 0, FAKE, None, cnt, None, 0, None) == 1
    assert L.dash_select(None, 10, 0, 0.5, 0.0, 0, 0, FAKE, None, cnt, None, 0, None) == 1
    need = L.dash_select_workspace_size(100000)
    assert need > 8 * 100000 and L.dash_select_workspace_size(-1) == 0
    assert L.dash_select(FAKE, 100000, 0, 0.5, 0.0, 0, 0, FAKE, None, cnt, None, 0, None) == 4    # no workspace
    assert L.dash_select(FAKE, 100000, 0, 0.5, 0.0, 0, 0, FAKE, None, cnt, FAKE, need - 1, None) == 4
    assert L.dash_score(FAKE, None, 10, 7, 0, FAKE, None) == 2
    assert L.dash_score(FAKE, None, 10, 64, 1, FAKE, None) == 1          # relative needs H
    assert L.dash_compact(FAKE, 10, FAKE, 5, 12, FAKE, None) == 2
    assert L.dash_linear(FAKE, 10, 100, FAKE, 128, FAKE, None) == 2      # K % 64
    assert L.dash_attention(FAKE, FAKE, FAKE, 10, 10, 4, 2, 96, None, None, FAKE, None) == 2
    assert L.dash_attention(FAKE, FAKE, FAKE, 20, 10, 4, 2, 64, None, None, FAKE, None) == 2  # M > T_kv causal

    # varlen: cu_seqlens must start at 0 and not decrease
    vcfg = dash.make_config(halt_layer=1)
    bad_cu = (ctypes.c_int32 * 3)(0, 10, 5)
    assert L.dash_prefill_varlen(ctypes.byref(dims), layers, FAKE, bad_cu, 2, ctypes.byref(vcfg), None, None, None,
                                 None, None, 0, None) == 1
    bad_cu0 = (ctypes.c_int32 * 3)(1, 10, 20)
    assert L.dash_prefill_varlen(ctypes.byref(dims), layers, FAKE, bad_cu0, 2, ctypes.byref(vcfg), None, None, None,
                                 None, None, 0, None) == 1
    ok_cu = (ctypes.c_int32 * 3)(0, 10, 20)
    assert L.dash_prefill_varlen(ctypes.byref(dims), layers, FAKE, ok_cu, 2, ctypes.byref(vcfg), None, None, None,
                                 None, None, 0, None) == 4   # valid layout, no workspace


def test_workspace_sizes_grow_with_tokens(L):
    dims = _dims()
    cfg = dash.make_config(halt_layer=2)
    sizes = [L.dash_prefill_workspace_size(ctypes.byref(dims), T, ctypes.byref(cfg)) for T in (1, 512, 4096)]
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    q = inputs.QWEN7B
    qd = dash.Dims(q.n_layers, q.d_model, q.n_heads, q.n_kv_heads, q.head_dim, q.ffn_dim, q.rms_eps, q.rope_theta)
    big = L.dash_prefill_workspace_size(ctypes.byref(qd), 32768, ctypes.byref(cfg))
    # activations for T = 32768 fit well inside one GPU's memory
    assert 1 << 30 < big < 8 << 30
    assert L.dash_layer_workspace_size(ctypes.byref(dims), 100, 50, 100) == 0  # T_kv < M rejected
    # a decode workspace sized for n sequences serves any fewer (3 or more add the
    # split-K partial sums of the tensor-core projections)
    dec = [L.dash_decode_workspace_size(ctypes.byref(qd), n) for n in range(1, 9)]
    assert all(0 < a <= b for a, b in zip(dec, dec[1:]))
    assert dec[2] - dec[1] > 8 << 20


def _cache_arr(n, k=FAKE, v=FAKE, cap=1024, ln=0):
    arr = (dash.KVCacheDesc * n)()
    for i in range(n):
        arr[i] = dash.KVCacheDesc(k, v, None, cap, ln)
    return arr


def test_kv_cache_and_decode_argument_errors(L):
    dims = _dims()
    layers = _fake_layers(4)
    cfg = dash.make_config(halt_layer=1, mode="prune", keep=0.5)
    K = ctypes.c_int64(0)
    pre = lambda caches, T=512, c=cfg: L.dash_prefill_kv(ctypes.byref(dims), layers, FAKE, T, ctypes.byref(c), None,
                                                         ctypes.byref(K), None, caches, None, 0, None)
    assert pre(None) == 1                                                  # caches required
    assert pre(_cache_arr(4, cap=511)) == 2                                # layer 0 holds T = 512 rows
    small = _cache_arr(4, cap=512)
    small[3].capacity = 255                                                # K = 256 rows after L_s
    assert pre(small) == 2
    small[3].capacity = 256
    assert pre(small) == 4                                                 # capacities fine, no workspace
    halt = dash.make_config(halt_layer=1, mode="halt", keep=0.5)
    assert pre(small, c=halt) == 2                                         # halt keeps T rows in every layer
    assert pre(_cache_arr(4, k=FAKE + 8)) == 1                             # misaligned cache
    assert pre(_cache_arr(4, ln=2000)) == 1                                # len > capacity
    # an empty prompt resets the lengths without touching the device
    emp = _cache_arr(4, ln=7)
    assert pre(emp, T=0) == 0 and [c.len for c in emp] == [0] * 4

    ws = L.dash_decode_workspace_size(ctypes.byref(dims), 2)
    assert ws > 0 and L.dash_decode_workspace_size(ctypes.byref(dims), 9) == 0
    pos = (ctypes.c_int32 * 2)(10, 20)
    dec = lambda n, caches, p=pos, w=None, wb=0: L.dash_decode_step(ctypes.byref(dims), layers, FAKE, n, p, caches,
                                                                     w, wb, None)
    assert dec(0, _cache_arr(8)) == 2                                      # no sequences
    assert dec(9, _cache_arr(36)) == 2                                     # more than DASH_DECODE_MAX_SEQ
    assert dec(2, None) == 1
    assert dec(2, _cache_arr(8), p=None) == 1
    assert dec(2, _cache_arr(8, cap=5, ln=5)) == 2                         # a full cache
    assert dec(2, _cache_arr(8, ln=3)) == 4                                # valid, no workspace
    assert dec(2, _cache_arr(8, ln=3), w=FAKE, wb=ws - 1) == 4             # one byte short
    neg = (ctypes.c_int32 * 2)(-1, 3)
    assert dec(2, _cache_arr(8), p=neg) == 1                               # negative position
    # decode attention op
    cs = _cache_arr(2, ln=100)
    att = lambda n, hq, hkv, hd, caches=cs, w=None, wb=0: L.dash_decode_attention(FAKE, n, caches, hq, hkv, hd, FAKE,
                                                                                  w, wb, None)
    assert att(2, 4, 2, 96) == 2                                           # head_dim
    assert att(2, 68, 2, 64) == 2                                          # group of 34 > 16
    assert att(9, 4, 2, 64) == 2                                           # too many sequences
    assert att(2, 4, 2, 64, caches=_cache_arr(2, ln=0)) == 2               # an empty cache
    assert att(2, 4, 2, 64) == 4                                           # no workspace
    assert L.dash_decode_attention_workspace_size(64) > 0 and L.dash_decode_attention_workspace_size(80) == 0


def test_binding_refuses_tensors_the_library_would_misread(L):
    """The binding passes raw pointers, so it checks each tensor first: a host
    tensor, another dtype, a strided view or a wrong shape raises ValueError
    before any library call (no GPU needed for these refusals)."""
    import torch
    bf = torch.zeros(8, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        dash.score(bf)                                   # host memory
    with pytest.raises(ValueError, match="CUDA"):
        dash.linear(bf, torch.zeros(16, 256, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        dash.compact(bf, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        dash.attention(bf, bf, bf, 2, 1, 128)
    with pytest.raises(ValueError, match="CUDA"):
        dash.select(torch.zeros(10))
    # dtype, stride and shape are checked the same way (shown on the helper itself)
    for bad, why in [(torch.zeros(4, 6), "float32"), (bf.t(), "strided"), (bf, "CUDA")]:
        with pytest.raises(ValueError, match=why):
            dash._t(bad, torch.bfloat16, "x")
    assert dash._t(None, torch.bfloat16, "x") is None
    with pytest.raises(ValueError, match="at least 9"):
        dash._out(torch.zeros(8, dtype=torch.int32), torch.int32, "idx_out", 9)
    # a stack takes its 16-bit format from its weights, all of one format
    w = {k: v.half() for k, v in inputs.make_layers(inputs.TINY, n_layers=1)[0].items()}
    st = dash.Stack(inputs.TINY, [w])
    assert st.dtype == torch.float16 and st.dims.dtype == 1
    mixed = dict(w, wo=w["wo"].bfloat16())
    with pytest.raises(ValueError, match="all float16"):
        dash.Stack(inputs.TINY, [mixed])
    with pytest.raises(ValueError, match="float16"):
        dash.prefill(st, bf, dash.make_config())         # bf16 hidden states for an fp16 stack


def test_headers_compile_and_link_as_plain_c(L, tmp_path):
    """The ABI is usable from C: both headers compile as strict C99, and a C
    program linked against libdash.so calls two host-only entry points."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi_user.c"
    src.write_text(
        '#include "dash.h"\n#include "dash_ops.h"\n#include <stdio.h>\n#include <string.h>\n'
        "int main(void) {\n"
        "  const char* s = dash_status_string(DASH_OK);\n"
        "  long long k = (long long)dash_topk_count(1000, 0.5, 64, 32);\n"
        '  printf("%s %lld\\n", s, k);\n'
        "  return (s != NULL && strlen(s) > 0 && k == 64 + 32 + 452) ? 0 : 1;\n"
        "}\n")
    exe = tmp_path / "abi_user"
    libdir = os.path.dirname(build.LIB)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", build.INCLUDE,
                        str(src), "-o", str(exe), "-L", libdir, "-l:libdash.so", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
