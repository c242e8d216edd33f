"""bench.py's host-side arithmetic (CPU only): the algorithmic bytes and flops the roofline
fractions divide by, the bound each record picks, and the traffic record written from an
ncu CSV and keyed on kernel sources."""
import json

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
    # the chunked form: three times the forward's chunk products
    assert bflops == 3 * bench.chunk_alg(W["lm1p3b_bf16"])[1]


def test_roofline_record_picks_the_slower_bound():
    hbm, tc = 6545.9, 1646.8
    r = bench.roofline_record(138_674_176, 23_622_320_128, 100e-6, hbm, tc, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - 138_674_176 / (hbm * 1e9) / 100e-6) < 1e-12
    assert abs(r["achieved"] / r["peak"] - r["frac"]) < 1e-12
    r = bench.roofline_record(1_000, 1e12, 1e-3, hbm, tc, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] / r["peak"] - r["frac"]) < 1e-12


CSV = """==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","(anonymous namespace)::ut_kernel(CUtensorMap_st, bf16)","1","7","(160, 1, 1)","(888, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","1,000"
"0","1","python","h","(anonymous namespace)::ut_kernel(CUtensorMap_st, bf16)","1","7","(160, 1, 1)","(888, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","10"
"1","1","python","h","void efla::<unnamed>::chunk_tc_kernel<0>(CUtensorMap_st)","1","7","(448, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Kbyte","2"
"1","1","python","h","void efla::<unnamed>::chunk_tc_kernel<0>(CUtensorMap_st)","1","7","(448, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","300"
"2","1","python","h","(anonymous namespace)::ut_kernel(CUtensorMap_st, bf16)","1","7","(160, 1, 1)","(888, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","5,000"
"2","1","python","h","(anonymous namespace)::ut_kernel(CUtensorMap_st, bf16)","1","7","(160, 1, 1)","(888, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","50"
"3","1","python","h","void efla::<unnamed>::chunk_tc_kernel<0>(CUtensorMap_st)","1","7","(448, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","7,000"
"3","1","python","h","void efla::<unnamed>::chunk_tc_kernel<0>(CUtensorMap_st)","1","7","(448, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","700"
"""


def test_traffic_record_is_written_from_the_ncu_csv_and_follows_the_sources(tmp_path, monkeypatch):
    h_fwd = bench.kernel_source_hash("efla_chunk_fwd")
    h_dec = bench.kernel_source_hash("efla_recurrent_step")
    assert h_fwd != h_dec and len(h_fwd) == 16
    csv = tmp_path / "dram.csv"
    csv.write_text(CSV)
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(tmp_path / "traffic.json"))
    rec = bench.traffic_from_csv(str(csv), "efla_chunk_fwd", calls=1)     # the last call only
    assert rec["bytes_per_call"] == 5_000 + 50 + 7_000 + 700 and rec["launches"] == 2
    rec = bench.traffic_from_csv(str(csv), "efla_chunk_fwd", calls=2)     # both calls, averaged
    assert rec["bytes_per_call"] == (1_010 + 2_300 + 5_050 + 7_700) // 2
    assert bench.ncu_traffic("efla_chunk_fwd") == rec["bytes_per_call"]
    assert bench.ncu_traffic("efla_backward") is None                    # not recorded
    assert rec["kernels"] == ["chunk_tc_kernel", "ut_kernel"]
    data = json.loads((tmp_path / "traffic.json").read_text())
    data["efla_recurrent_step"] = dict(rec, kernel_source="0000000000000000")
    (tmp_path / "traffic.json").write_text(json.dumps(data))
    assert bench.ncu_traffic("efla_recurrent_step") is None              # recorded for other sources


def test_cotangents_are_seeded():
    w = W["tiny_fp32"].replace(T=17)
    a, b = workloads.make_cotangents(w), workloads.make_cotangents(w)
    assert (a["dO"] == b["dO"]).all() and (a["dS_T"] == b["dS_T"]).all()
    assert workloads.make_cotangents(w, with_state_grad=False)["dS_T"] is None


CSV_BWD = """"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","void efla::<unnamed>::chunk_tc_kernel<0, 1>(CUtensorMap_st)","1","7","(448, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","9,000"
"1","1","python","h","void efla::<unnamed>::bwd_chain_kernel(CUtensorMap_st)","1","7","(320, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","3,000"
"1","1","python","h","void efla::<unnamed>::bwd_chain_kernel(CUtensorMap_st)","1","7","(320, 1, 1)","(128, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","300"
"2","1","python","h","void efla::<unnamed>::bwd_tile_kernel(CUtensorMap_st)","1","7","(256, 1, 1)","(2048, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","4,000"
"2","1","python","h","void efla::<unnamed>::bwd_tile_kernel(CUtensorMap_st)","1","7","(256, 1, 1)","(2048, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","400"
"""


def test_saved_backward_traffic_counts_only_its_own_kernels(tmp_path, monkeypatch):
    """The saved-residual backward runs the reverse chain and the per-chunk kernel only: a
    forward launch in the same log (the one that saved the residuals) is not counted, and the
    record follows its own, smaller set of kernel sources."""
    csv = tmp_path / "dram.csv"
    csv.write_text(CSV_BWD)
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(tmp_path / "traffic.json"))
    rec = bench.traffic_from_csv(str(csv), "efla_backward_saved", calls=1)
    assert rec["bytes_per_call"] == 3_000 + 300 + 4_000 + 400 and rec["launches"] == 2
    assert rec["kernels"] == ["bwd_chain_kernel", "bwd_tile_kernel"]
    assert bench.ncu_traffic("efla_backward_saved") == rec["bytes_per_call"]
    assert set(bench.KERNEL_SOURCES["efla_backward_saved"]) < set(bench.KERNEL_SOURCES["efla_backward"])
