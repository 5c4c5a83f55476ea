"""Host-side measurement logic (no GPU): the algorithmic work counts behind
every reported FLOP rate and bound, and the bench's traffic bookkeeping.

The expected totals are the hand-derived figures of the workloads (parameter
counts written out matrix by matrix; causal attention as 4*hq*hd FLOPs per
visible pair), not values produced by the code under test."""
import hashlib
import json
import os

import pytest

from long_context_prefill_tcgen05_b200 import costs, inputs

QWEN, LLAMA = inputs.QWEN7B, inputs.LLAMA8B


def _qwen_params_per_layer():
    d, f = 3584, 18944
    q, kv = 28 * 128, 4 * 128
    return d * q + d * kv + d * kv + q * d + d * f + d * f + f * d   # wq wk wv wo wg wu wd


def test_linear_flops_are_two_per_weight():
    assert _qwen_params_per_layer() == 233_046_016
    assert costs.linear_flops_per_token(QWEN) == 2 * 233_046_016          # 466.1 MFLOP per token and layer
    d, f, q, kv = 4096, 14336, 32 * 128, 8 * 128
    assert costs.linear_flops_per_token(LLAMA) == 2 * (d * (q + 2 * kv) + q * d + 3 * d * f)


def test_layer_weight_bytes_are_bf16_weights_plus_two_gains():
    assert costs.layer_weight_bytes(QWEN) == 2 * _qwen_params_per_layer() + 2 * 2 * 3584


def test_attention_flops_per_visible_pair():
    assert costs.causal_pairs(1) == 1 and costs.causal_pairs(4) == 10
    assert costs.attn_flops(QWEN, 1) == 4 * 28 * 128
    # 2 * d * T^2 per layer at full length (the T^2/2 pairs times 4*hq*hd)
    T = 32768
    assert costs.attn_flops(QWEN, costs.causal_pairs(T)) == 2 * 3584 * T * (T + 1)


@pytest.mark.parametrize("mode,K,tflop", [("dense", None, 643.2), ("prune", 16384, 428.6)])
def test_qwen_32k_totals(mode, K, tflop):
    got = costs.prefill_flops(QWEN, 32768, 11, K, mode) / 1e12
    assert abs(got - tflop) < 0.05


@pytest.mark.parametrize("mode,K,tflop", [("dense", None, 5158.7), ("halt", int(0.3 * 131072), 3106.0)])
def test_qwen_128k_totals_with_evenly_spread_active_rows(mode, K, tflop):
    got = costs.prefill_flops(QWEN, 131072, 11, K, mode) / 1e12
    assert abs(got - tflop) < 0.05


def test_llama_varlen_totals():
    cu = [0, 16384, 32768, 49152, 65536]
    dense = costs.varlen_prefill_flops(LLAMA, cu) / 1e12
    pruned = costs.varlen_prefill_flops(LLAMA, cu, 13, [int(0.4 * 16384)] * 4, "prune") / 1e12
    assert abs(dense - 1196.3) < 0.05
    assert abs(pruned - 754.5) < 0.05
    assert abs(dense / pruned - 1.585) < 0.001


def test_keeping_every_token_costs_the_dense_prefill():
    T = 4096
    dense = costs.prefill_flops(QWEN, T)
    assert costs.prefill_flops(QWEN, T, 11, T, "prune") == dense
    assert costs.prefill_flops(QWEN, T, 11, T, "halt", active_idx=range(T)) == dense


def test_halt_counts_the_keys_each_active_query_sees():
    T, idx = 1000, [0, 10, 999]
    lin = costs.linear_flops_per_token(QWEN)
    full = T * lin + costs.attn_flops(QWEN, costs.causal_pairs(T))
    late = 3 * lin + costs.attn_flops(QWEN, 1 + 11 + 1000) + (T - 3) * 2 * 3584 * 2 * 512
    assert costs.prefill_flops(QWEN, T, 11, 3, "halt", active_idx=idx) == 12 * full + 16 * late


def test_launch_work_units():
    assert costs.launch_work({"kind": "gemm_qkv_rope", "m": 3, "n": 5, "k": 7}, QWEN) == ("flop", 210)
    assert costs.launch_work({"kind": "attention", "m": 4, "n": 4, "k": 10}, QWEN) == ("flop", 10 * 4 * 28 * 128)
    assert costs.launch_work({"kind": "attention", "m": 4, "n": 9, "k": -1}, QWEN, {4: 7}) == ("flop", 7 * 4 * 28 * 128)
    assert costs.launch_work({"kind": "rmsnorm", "m": 10, "n": 3584, "k": 0}, QWEN) == ("byte", 2 * 10 * 3584 * 2)


def test_recorded_traffic_scales_by_rows_and_expires_with_the_source(tmp_path, monkeypatch):
    import bench
    (tmp_path / "profiles").mkdir()
    src_dir = tmp_path / "long_context_prefill_tcgen05_b200" / "csrc"
    src_dir.mkdir(parents=True)
    src = src_dir / "attention.cuh"
    src.write_bytes(b"// kernel v1\n")
    rec = {"attention": {"src_sha256": hashlib.sha256(b"// kernel v1\n").hexdigest(), "rows": 1000,
                         "bytes_per_launch": 5000, "source": "x", "scales_with": "rows"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    recs = [{"kind": "attention", "m": 1000}, {"kind": "attention", "m": 500}, {"kind": "gemm_resid", "m": 9}]
    assert bench.recorded_traffic("attention", recs) == pytest.approx((5000 + 2500) / 2)
    src.write_bytes(b"// kernel v2\n")
    assert bench.recorded_traffic("attention", recs) is None
    assert bench.recorded_traffic("gemm", recs) is None


def test_committed_traffic_record_names_an_existing_capture():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "traffic.json")) as f:
        rec = json.load(f)["attention"]
    assert os.path.exists(os.path.join(root, rec["source"]))
    with open(os.path.join(root, rec["source"])) as f:
        assert rec["src_sha256"] in f.read()
