"""GPU parity at the edges of the accepted scale range.

The header accepts any finite scale >= 0.  At scale 0 every visible key gets
the same weight, so each output row is the mean of the visible V rows (the
closed form the oracle is pinned to); a tiny positive scale (1e-30) must
behave the same way to within rounding.  Each path — prefill (causal and
not, both head sizes, tiles crossing the diagonal and the sequence end),
decode with split-KV merges, a mixed batch, and small-seq — is compared with
the fp64 oracle at the usual tolerances."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, oracle_varlen, run_varlen

pytestmark = pytest.mark.gpu

SCALES = [0.0, 1e-30]


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def build(lens, qlens, hq, hkv, d, causal, scale, seed):
    return workloads.build_varlen_case("scale", lens, qlens, hq, hkv, d, causal, seed,
                                       scale=scale)


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [128, 64])
def test_prefill_scale_edges(scale, causal, d):
    lens = [2, 17, 129, 300, 513]
    cpu = build(lens, lens, 8, 2, d, causal, scale, seed=d + int(causal))
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"prefill scale={scale} d={d}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("scale", SCALES)
def test_chunked_prefill_scale_edges(scale):
    cpu = build([600, 333, 129, 1000], [100, 333, 2, 130], 16, 2, 128, True, scale, seed=5)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"chunked scale={scale}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("scale", SCALES)
def test_decode_scale_edges(scale):
    lens = [1, 15, 16, 17, 255, 700, 2049, 5000]
    cpu = build(lens, [1] * len(lens), 32, 8, 128, True, scale, seed=7)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"decode scale={scale}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("scale", SCALES)
def test_mixed_scale_edges(scale):
    lens = [700, 40, 300, 1, 2000, 17, 5, 129]
    qlens = [64, 1, 300, 1, 1, 17, 1, 100]
    cpu = build(lens, qlens, 16, 2, 128, True, scale, seed=11)
    out, _, _, ws = run_varlen(case_to(cpu, "cuda"))
    assert_attention_close(out, oracle_varlen(cpu), what=f"mixed scale={scale}")
    assert pa.get_error(ws) == (0, 0)


@pytest.mark.parametrize("scale", SCALES)
def test_scale_zero_prefill_row_is_mean_of_visible_values(scale):
    # the closed form directly on the GPU output: row i of a causal prefill
    # over L keys is the mean of V rows 0..i of its KV head
    cpu = build([200], [200], 4, 4, 128, True, scale, seed=3)
    out, _, _, _ = run_varlen(case_to(cpu, "cuda"))
    v = cpu.v_logical.double()
    mean = torch.cumsum(v, 0) / torch.arange(1, 201, dtype=torch.float64)[:, None, None]
    err = (out.double().cpu() - mean).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3


def _smallseq(case):
    out = torch.full_like(case.q, float("nan"))
    ws = pa.error_workspace()
    pa.attention_smallseq(case.q, case.k, case.v, case.cu_seqlens_kv, case.scale, out,
                          max_seqlen_kv=16, workspace=ws)
    torch.cuda.synchronize()
    return out, ws


@pytest.mark.parametrize("scale", SCALES)
def test_smallseq_scale_edges(scale):
    rng = np.random.default_rng(4)
    lens = rng.integers(0, 17, size=500).tolist()
    lens[:3] = [0, 1, 16]
    cpu = workloads.build_smallseq_case("scale", lens, 16, 16, 128, seed=4, scale=scale)
    out, ws = _smallseq(case_to(cpu, "cuda"))
    ref = oracle.attention_smallseq(workloads.bf16_bits(cpu.q), workloads.bf16_bits(cpu.k),
                                    workloads.bf16_bits(cpu.v), cpu.cu_seqlens_kv.numpy(),
                                    cpu.num_kv_heads, scale)
    assert_attention_close(out, ref, what=f"smallseq scale={scale}")
    assert pa.get_error(ws) == (0, 0)
