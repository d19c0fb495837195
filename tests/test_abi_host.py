"""CPU-only checks of the C ABI: the library builds, loads and exports every
symbol include/pa.h declares, and host-visible argument errors are rejected
before anything is launched (no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest
import torch

import paged_kv_gqa_reshape_b200 as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    with open(os.path.join(ROOT, "include", "pa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_exported_set():
    assert declared_symbols() == sorted(pa.EXPORTED_SYMBOLS)


def test_library_loads_and_exports_every_declared_symbol():
    lib = pa.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version():
    assert pa.status_string(0) == "PA_OK"
    for s in range(1, 6):
        assert pa.status_string(s).startswith("PA_ERR_")
    assert "sm_100a" in pa.version()


def test_workspace_size_is_a_function_of_the_arguments():
    a = pa.varlen_workspace_size(64, 64, 32, 8, 128)
    b = pa.varlen_workspace_size(64, 64, 32, 8, 128)
    assert a == b and a > 256
    assert pa.varlen_workspace_size(256, 4344, 64, 8, 128) > a
    assert pa.varlen_workspace_size(-1, 1, 1, 1, 64) == 0


def _varlen(lib, **over):
    args = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, bt=1 << 12, mb=4, sl=1 << 12, qsl=1 << 12,
                S=2, T=4, Hq=4, Hkv=2, D=64, BS=16, NB=8, mql=4, msl=64, scale=0.125,
                causal=1, out=1 << 12, ws=1 << 12, wsb=1 << 30, stream=None)
    args.update(over)
    return lib.pa_attention_varlen(*args.values())


@pytest.mark.parametrize("over,expect", [
    (dict(Hq=6, Hkv=4), 1),           # Hq % Hkv != 0
    (dict(Hkv=0), 1),
    (dict(D=96), 2),                  # unsupported head_dim
    (dict(BS=24), 2),                 # block size not a multiple of 16
    (dict(BS=8), 2),
    (dict(BS=1024), 2),               # above the largest block size
    (dict(Hq=258, Hkv=2), 2),         # GQA group > 128
    (dict(causal=2), 1),
    (dict(scale=float("nan")), 1),
    (dict(scale=-0.125), 1),          # negative scale
    (dict(q=0), 1),                   # null pointer
    (dict(q=(1 << 12) + 2), 1),       # misaligned
    (dict(wsb=16), 1),                # workspace too small
    (dict(NB=0), 1),
])
def test_varlen_rejects_before_launch(over, expect):
    assert _varlen(pa.load(), **over) == expect


def test_varlen_empty_batch_is_a_no_op():
    assert _varlen(pa.load(), S=0) == 0
    assert _varlen(pa.load(), T=0) == 0


def _spans(lib, **over):
    args = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, bt=1 << 12, mb=4, sl=1 << 12, qsl=1 << 12,
                S=2, T=4, Hq=4, Hkv=2, D=64, BS=16, NB=8, mql=4, msl=64, scale=0.125,
                so=1 << 12, sp=1 << 12, nsp=2, out=1 << 12, ws=1 << 12, wsb=1 << 30, stream=None)
    args.update(over)
    return lib.pa_attention_varlen_spans(*args.values())


@pytest.mark.parametrize("over,expect", [
    (dict(so=0), 1),                  # span offsets are required
    (dict(sp=0), 1),                  # spans required when there are some
    (dict(nsp=-1), 1),
    (dict(so=(1 << 12) + 2), 1),      # misaligned int32
    (dict(D=96), 2),
    (dict(wsb=16), 1),
])
def test_varlen_spans_rejects_before_launch(over, expect):
    assert _spans(pa.load(), **over) == expect


def test_varlen_spans_empty_batch_is_a_no_op():
    assert _spans(pa.load(), S=0, so=0) == 0
    assert _spans(pa.load(), T=0) == 0


def test_ex_entry_points_check_stride_and_dtype():
    lib = pa.load()
    base = dict(k=1 << 12, v=1 << 12, sm=1 << 12, T=4, Hkv=2, D=64, kc=1 << 12, vc=1 << 12,
                NB=8, BS=16, stride=0, dtype=0, ws=None, stream=None)

    def wkv(**over):
        a = dict(base)
        a.update(over)
        return lib.pa_write_kv_ex(*a.values())
    assert wkv(stride=16 * 2 * 64 - 8) == 1        # smaller than one block
    assert wkv(stride=2 * 16 * 2 * 64 + 4) == 1    # not a multiple of 8 elements
    assert wkv(dtype=7) == 1
    assert wkv(T=0) == 0
    args = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, bt=1 << 12, mb=4, sl=1 << 12, qsl=1 << 12,
                S=2, T=4, Hq=4, Hkv=2, D=64, BS=16, NB=8, stride=0, dtype=0, mql=4, msl=64,
                scale=0.125, causal=1, so=None, sp=None, nsp=0, out=1 << 12, ws=1 << 12,
                wsb=1 << 30, stream=None)

    def var(**over):
        a = dict(args)
        a.update(over)
        return lib.pa_attention_varlen_ex(*a.values())
    assert var(stride=100) == 1
    assert var(dtype=5) == 1
    assert var(S=0) == 0


def test_write_kv_rejects_before_launch():
    lib = pa.load()
    ok = dict(k=1 << 12, v=1 << 12, sm=1 << 12, T=3, Hkv=2, D=64, kc=1 << 12, vc=1 << 12,
              NB=4, BS=16, ws=None, stream=None)
    for over in (dict(D=60), dict(Hkv=0), dict(NB=0), dict(k=0), dict(kc=(1 << 12) + 8),
                 dict(T=-1)):
        a = dict(ok)
        a.update(over)
        assert lib.pa_write_kv(*a.values()) == 1, over
    a = dict(ok)
    a["T"] = 0
    assert lib.pa_write_kv(*a.values()) == 0


def test_smallseq_rejects_before_launch():
    lib = pa.load()
    ok = dict(q=1 << 12, k=1 << 12, v=1 << 12, cu=1 << 12, B=4, Hq=4, Hkv=4, D=128, mx=16,
              scale=0.1, out=1 << 12, ws=None, stream=None)
    for over, expect in ((dict(mx=17), 2), (dict(D=80), 2), (dict(Hq=6), 1), (dict(cu=0), 1),
                         (dict(out=(1 << 12) + 4), 1)):
        a = dict(ok)
        a.update(over)
        assert lib.pa_attention_smallseq(*a.values()) == expect, over
    a = dict(ok)
    a["B"] = 0
    assert lib.pa_attention_smallseq(*a.values()) == 0


def test_python_binding_rejects_cpu_and_wrong_dtypes():
    q = torch.zeros(4, 4, 64, dtype=torch.bfloat16)
    kc = torch.zeros(8, 16, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pa.attention_varlen(q, kc, kc, torch.zeros(2, 2, dtype=torch.int32),
                            torch.zeros(2, dtype=torch.int32), torch.zeros(3, dtype=torch.int32),
                            2, 0.1, True, q)
    with pytest.raises(TypeError):
        pa.write_kv(q.float(), q, torch.zeros(4, dtype=torch.int64), kc, kc)


def test_python_binding_device_agreement():
    # every tensor of a call must sit on the device its kernels run on
    a, b = torch.zeros(1), torch.zeros(1, device="meta")
    pa._same_device(torch.device("cpu"), x=a, y=None)
    with pytest.raises(ValueError, match="y is on meta"):
        pa._same_device(torch.device("cpu"), x=a, y=b)


def test_struct_layouts_match_the_header(tmp_path):
    # the C structs of include/pa.h, laid out by the C compiler, against the
    # ctypes mirrors the binding passes by pointer
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "pa.h"\n'
        'int main(void) {\n'
        '  printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(pa_score_mods),\n'
        '         offsetof(pa_score_mods, alibi_slopes), offsetof(pa_score_mods, mask),\n'
        '         offsetof(pa_score_mods, mask_len), sizeof(pa_strides),\n'
        '         offsetof(pa_strides, cache_head));\n'
        '  return 0;\n}\n')
    exe = tmp_path / "layout"
    import subprocess
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    want = [ctypes.sizeof(pa._ScoreMods), pa._ScoreMods.alibi_slopes.offset,
            pa._ScoreMods.mask.offset, pa._ScoreMods.mask_len.offset, ctypes.sizeof(pa._Strides),
            pa._Strides.cache_head.offset]
    assert got == want


def _mods_call(lib, strides=None, mods=None, **over):
    a = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, bt=1 << 12, mb=4, sl=1 << 12, qsl=1 << 12,
             S=2, T=4, Hq=4, Hkv=2, D=64, BS=16, NB=8, dtype=0, mql=4, msl=64, scale=0.125,
             causal=1, so=None, sp=None, nsp=0)
    a.update(over)
    return lib.pa_attention_varlen_mods(
        *a.values(), ctypes.byref(strides) if strides is not None else None,
        ctypes.byref(mods) if mods is not None else None, 1 << 12, 1 << 12, 1 << 30, None)


def test_varlen_mods_rejects_layouts_and_modifiers_before_launch():
    lib = pa.load()
    S = pa._Strides
    # q: head stride below D with a token stride that is not head-major either
    assert _mods_call(lib, S(64, 32, 0, 0, 0, 0, 0)) == 2
    # q stride not a multiple of 8 elements
    assert _mods_call(lib, S(4 * 64 + 4, 64, 0, 0, 0, 0, 0)) == 1
    # cache: overlapping head rows, then a block stride smaller than a block
    assert _mods_call(lib, S(0, 0, 0, 0, 16 * 96, 96, 32)) == 2
    assert _mods_call(lib, S(0, 0, 0, 0, 8, 2 * 64, 64)) == 1
    # head-major cache with a block stride short of its extent
    assert _mods_call(lib, S(0, 0, 0, 0, 2 * 16 * 64 - 8, 64, 16 * 64)) == 1
    M = pa._ScoreMods
    assert _mods_call(lib, None, M(-1.0, None, None, 0, 0, 0)) == 1            # negative cap
    assert _mods_call(lib, None, M(float("inf"), None, None, 0, 0, 0)) == 1
    assert _mods_call(lib, None, M(0.0, (1 << 12) + 2, None, 0, 0, 0)) == 1    # slopes misaligned
    assert _mods_call(lib, None, M(0.0, None, (1 << 12) + 4, 0, 64, 64)) == 1  # mask misaligned
    assert _mods_call(lib, None, M(0.0, None, 1 << 12, 0, 66, 64)) == 1        # row stride % 4
    assert _mods_call(lib, None, M(0.0, None, 1 << 12, 0, 64, 0)) == 1         # mask_len 0
    assert _mods_call(lib, None, M(0.0, None, None, 0, 0, 0), S=0) == 0       # empty batch
    # a modifier with scale 0 (the kernels work in unscaled-score units)
    assert _mods_call(lib, None, M(30.0, None, None, 0, 0, 0), scale=0.0) == 1
    assert _mods_call(lib, None, M(0.0, 1 << 12, None, 0, 0, 0), scale=0.0) == 1
    assert _mods_call(lib, None, M(0.0, None, 1 << 12, 0, 64, 64), scale=0.0) == 1


def test_write_kv_strided_rejects_before_launch():
    lib = pa.load()
    S = pa._Strides

    def wkv(strides, **over):
        a = dict(k=1 << 12, v=1 << 12, sm=1 << 12, T=4, Hkv=2, D=64, kc=1 << 12, vc=1 << 12,
                 NB=8, BS=16)
        a.update(over)
        return lib.pa_write_kv_strided(*a.values(), ctypes.byref(strides), 0, None, None)
    assert wkv(S(0, 0, 0, 0, 16 * 96, 96, 32)) == 2       # overlapping rows
    assert wkv(S(0, 0, 0, 0, 2 * 16 * 64, 64, 16 * 64 + 4)) == 1
    assert wkv(S(0, 0, 0, 0, 2 * 16 * 64, 64, 16 * 64), D=48) == 2   # D/8 not a power of two
    assert wkv(S(0, 0, 0, 0, 2 * 16 * 64, 64, 16 * 64), T=0) == 0


def test_smallseq_bwd_rejects_before_launch():
    lib = pa.load()

    def bwd(**over):
        a = dict(q=1 << 12, k=1 << 12, v=1 << 12, do=1 << 12, w=1 << 12, wl=16, cu=1 << 12,
                 B=4, Hq=4, Hkv=2, D=128, mx=16, scale=0.1, dtype=0, dq=1 << 12, dk=1 << 12,
                 dv=1 << 12, ws=None, stream=None)
        a.update(over)
        return lib.pa_attention_smallseq_bwd(*a.values())
    assert bwd(mx=17) == 2
    assert bwd(Hq=34, Hkv=2) == 2        # 17 query heads per KV head
    assert bwd(wl=0) == 1
    assert bwd(w=(1 << 12) + 1) == 1
    assert bwd(dk=(1 << 12) + 8) == 1
    assert bwd(D=96) == 2
    assert bwd(B=0) == 0
