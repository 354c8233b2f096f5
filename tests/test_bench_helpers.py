"""Host-side helpers of bench.py (no GPU)."""
import numpy as np

import bench
import oracle


def test_causal_mask_words_keep_every_causal_block():
    # the dense reference of the bench keeps every block j <= i, in the ABI's
    # bit layout (word j // 32, bit j % 32), nothing above the diagonal
    for nb in (1, 31, 32, 33, 100, 257):
        words = (nb + 31) // 32
        got = bench.causal_mask_words(nb, words).numpy().view(np.uint32)
        ref = oracle.pack_mask(np.tril(np.ones((1, 1, nb, nb), dtype=bool)))[0, 0]
        assert got.shape == (nb, words)
        assert np.array_equal(got, ref), nb


_CSV = """==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","prism::estimator_kernel(prism::EstParams, prism::TermMaps)","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","1000"
"0","1","python","h","prism::estimator_kernel(prism::EstParams, prism::TermMaps)","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","10"
"1","1","python","h","prism::attn::sparse_attn_kernel(CUtensorMap, CUtensorMap)","1","7","(384, 1, 1)","(4096, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","2"
"1","1","python","h","prism::attn::sparse_attn_kernel(CUtensorMap, CUtensorMap)","1","7","(384, 1, 1)","(4096, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","500"
"2","1","python","h","prism::estimator_kernel(prism::EstParams, prism::TermMaps)","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","3000"
"2","1","python","h","prism::estimator_kernel(prism::EstParams, prism::TermMaps)","1","7","(512, 1, 1)","(148, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","30"
"""


def test_traffic_record_roundtrip_and_staleness(tmp_path, monkeypatch):
    csv = tmp_path / "cap.csv"
    csv.write_text(_CSV)
    out = tmp_path / "dram_traffic.json"
    bench.record_traffic([str(csv)], "llama3_8b_32k", {"llama3_8b_128k": 4.0}, str(out))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(out))
    got = bench.profiled_traffic("llama3_8b_32k")
    assert got == {"estimator_kernel": 2020.0, "sparse_attn_kernel": 2000500.0}  # mean of two launches
    assert bench.profiled_traffic("llama3_8b_128k") == {"estimator_kernel": 8080.0, "sparse_attn_kernel": 8002000.0}
    assert bench.profiled_traffic("sweep_8k") == {}  # no factor recorded for it
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.profiled_traffic("llama3_8b_32k") == {}  # sources changed since the capture


def test_oracle_sample_spreads_over_groups_and_blocks():
    from tests import gen
    w = gen.WORKLOADS["llama3_8b_128k"]
    heads, blocks = bench.sample_heads_and_blocks(w, seed=3)
    assert len(heads) == 4 and sorted({h // 4 for h in heads}) == [0, 2, 5, 7]
    assert len(blocks) == 16 and {0, 1, w.nb // 2, w.nb - 1} <= set(blocks)
    tiny = gen.WORKLOADS["tiny_2k"]
    heads, blocks = bench.sample_heads_and_blocks(tiny, seed=0)
    assert heads == [0] and blocks == list(range(16))
