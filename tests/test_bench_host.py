"""bench.py's host-side arithmetic (CPU only): the algorithmic bytes and flops the roofline
fractions divide by, the fp32 ALU peak, and the traffic lookup keyed on kernel sources."""
import os

import bench
import workloads

W = workloads.CHUNK_WORKLOADS


def test_forward_algorithmic_bytes_and_flops():
    """B4 H16 T2048 d128 bf16: read q, k, v (2 B x 128 each), beta (2 B), write o (2 B x 128)
    per token and head, plus S_T (fp32 128 x 128 per head); per chunk 5 x 2 C^2 d + 3 x 2 C d^2."""
    nbytes, flops = bench.chunk_alg(W["lm1p3b_bf16"])
    token_heads = 4 * 16 * 2048
    assert nbytes == token_heads * (4 * 128 * 2 + 2) + 64 * 128 * 128 * 4 == 138_674_176
    assert flops == 64 * 32 * (5 * 2 * 64 * 64 * 128 + 3 * 2 * 64 * 128 * 128) == 23_622_320_128
    # with an initial state given, S0 is read too
    nb_long, _ = bench.chunk_alg(W["longctx_bf16"])
    assert nb_long == 16 * 32768 * (4 * 128 * 2 + 2) + 2 * 16 * 128 * 128 * 4


def test_decode_and_backward_algorithmic_counts():
    dbytes, dflops = bench.decode_alg(workloads.DECODE_WORKLOAD)
    assert dbytes == 256 * 16 * (2 * 128 * 128 * 4 + (4 * 128 + 1) * 4)
    assert dflops == 256 * 16 * 6 * 128 * 128
    bbytes, bflops = bench.backward_alg(W["lm1p3b_bf16"])
    token_heads = 4 * 16 * 2048
    # read q, k, v, dO (bf16) and beta; write dq, dk, dv (fp32) and dbeta; dS0 per head
    assert bbytes == token_heads * (4 * 128 * 2 + 2 + 3 * 128 * 4 + 4) + 64 * 128 * 128 * 4
    assert bflops == token_heads * 18 * 128 * 128


def test_fp32_alu_peak():
    assert abs(bench.fp32_alu_peak_tflops() - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9


def test_traffic_lookup_follows_the_entry_points_sources(tmp_path, monkeypatch):
    h_fwd = bench.kernel_source_hash("efla_chunk_fwd")
    h_dec = bench.kernel_source_hash("efla_recurrent_step")
    assert h_fwd != h_dec and len(h_fwd) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.md").write_text(
        f"traffic|efla_chunk_fwd|111|{h_fwd}\ntraffic|efla_recurrent_step|222|0000000000000000\n")
    csrc = os.path.join(bench.ROOT, "delta_rule_linear_02_b200")
    os.symlink(csrc, tmp_path / "delta_rule_linear_02_b200")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("efla_chunk_fwd") == 111
    assert bench.ncu_traffic("efla_recurrent_step") is None      # recorded for other sources
    assert bench.ncu_traffic("efla_backward") is None            # not recorded


def test_cotangents_are_seeded():
    w = W["tiny_fp32"].replace(T=17)
    a, b = workloads.make_cotangents(w), workloads.make_cotangents(w)
    assert (a["dO"] == b["dO"]).all() and (a["dS_T"] == b["dS_T"]).all()
    assert workloads.make_cotangents(w, with_state_grad=False)["dS_T"] is None
