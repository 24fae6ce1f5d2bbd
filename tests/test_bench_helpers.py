"""Host-side pieces of bench.py that decide what the JSON line reports (no GPU)."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_only_while_the_profiled_source_is_unchanged(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "decode_gateup_traffic.json")))
    sha = hashlib.sha256(open(bench.GATEUP_SRC, "rb").read()).hexdigest()
    same = rec.get("source_sha256") == sha and rec.get("kernel") == bench.GATEUP_KERNEL
    want = rec["bytes_per_launch"] if same else None
    assert bench.gateup_traffic() == want
    changed = tmp_path / "decode_gemv.cuh"
    changed.write_bytes(open(bench.GATEUP_SRC, "rb").read() + b"// changed")
    monkeypatch.setattr(bench, "GATEUP_SRC", str(changed))
    assert bench.gateup_traffic() is None  # counters taken on another version of the kernel: no traffic


def test_algorithmic_bytes_of_the_decode_workload():
    from bit_quantized_moe_02_b200 import synth
    wl = synth.WORKLOADS["decode"]
    s = wl.shape
    # routed IQ2X gate + up (66 B / 256 weights) + shared bf16 gate + up + x (bf16)
    want = s.k * 2 * s.f * s.d // 256 * 66 + 2 * s.f_shared * s.d * 2 + s.d * 2
    assert bench.gateup_bytes(wl) == want == 68165632


def test_step_bytes_counts_each_touched_expert_once():
    from bit_quantized_moe_02_b200 import synth
    s = synth.WORKLOADS["decode"].shape
    q4 = synth.WORKLOADS["q4"].shape
    # per expert: IQ2X gate and up [2048 x 4096] at 66 B per 256 weights, Q2K down [4096 x 2048] at 84 B
    assert s.expert_bytes == 2 * 2048 * 16 * 66 + 4096 * 8 * 84 == 7077888
    assert q4.expert_bytes == 3 * 2048 * 4096 // 256 * 144 == 14155776
    fixed = s.shared_bytes + s.router_bytes
    assert bench.step_bytes(s, 0, 0) == fixed == 3 * 2048 * 4096 * 2 + 256 * 4096 * 2
    assert bench.step_bytes(s, 24, 4) - bench.step_bytes(s, 23, 4) == s.expert_bytes
    assert bench.step_bytes(s, 24, 5) - bench.step_bytes(s, 24, 4) == 4096 * (2 + 4)
    # the B = 1 decode workload touches k experts: the same bytes as the main line's per-token figure
    assert bench.step_bytes(s, s.k, 1) == bench.layer_bytes(synth.WORKLOADS["decode"])


def test_every_other_workload_gets_its_own_oracle_baseline(monkeypatch):
    """workload_cpu_baselines times the oracle on each workload's own layer with a bounded per-thread sample and
    reports it in the contract's cpu_baseline form (value, unit, cores, kind, sample)."""
    calls = []

    def fake(wl, n_tokens, nthreads, seed_stream=7):
        calls.append((wl.name, n_tokens, nthreads))
        return 10.0 * n_tokens, 0.1

    monkeypatch.setattr(bench, "oracle_tokens_per_s", fake)
    res = bench.workload_cpu_baselines(4)
    assert set(res) == {"tiny", "batched", "prefill", "q4"}
    for name, cb in res.items():
        assert cb["kind"] == "oracle" and cb["cores"] == 4 and cb["unit"] == bench.UNIT
        assert cb["value"] > 0 and name in cb["sample"]
    assert [c[0] for c in calls] == ["tiny", "batched", "prefill", "q4"]
    assert all(nthreads == 4 and n % 4 == 0 for _, n, nthreads in calls)
