"""Host logic around the kernels, no GPU: the ncu traffic summary that the
benchmark's roofline reports, and the Python binding's argument checks that
run before any call into the library."""
import json

import numpy as np
import pytest
import torch

from nvfp4_block_scaled_gemm_b200 import profile_case, synth
from nvfp4_block_scaled_gemm_b200.build import source_hash

HEADER = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
          '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')


def ncu_rows(launch_id, kernel, read, write, us):
    rows = []
    for name, unit, val in (("dram__bytes_read.sum", "byte", read), ("dram__bytes_write.sum", "Kbyte", write),
                            ("gpu__time_duration.sum", "usecond", us)):
        rows.append(f'"{launch_id}","1","python","h","{kernel}","1","7","(128, 1, 1)","(8, 1, 1)","0","10.0",'
                    f'"Command line profiler metrics","{name}","{unit}","{val}"\n')
    return rows


def test_traffic_summary_takes_the_last_launch_of_each_shape(tmp_path):
    shapes = synth.ATTN_SWEEP_M
    lines = ["==PROF== Connected to process 1\n", HEADER]
    lid = 0
    for i, m in enumerate(shapes):
        kernel = "void nvfp4_gemv_kernel<1, 1>(GemvParams)" if m == 1 else "void nvfp4_gemm_kernel<16>(x)"
        for it in range(2):
            # the first launch of a shape carries junk; the summary must use the second
            lines += ncu_rows(lid, kernel, 1_000_000 * (i + 1) + (0 if it else 999), 2.5 * it, 10.0 + i)
            lid += 1
        lines += ncu_rows(lid, "void other_kernel(int)", 5, 5, 1.0)   # not a GEMM launch: ignored
        lid += 1
    csv_path = tmp_path / "t.csv"
    csv_path.write_text("".join(lines))
    out = tmp_path / "t.json"
    rec = profile_case.summarize_traffic(str(csv_path), str(out), iters=2)
    assert rec == json.loads(out.read_text())
    assert rec["per_shape_dram_read"] == {f"M{m}": 1_000_000 * (i + 1) for i, m in enumerate(shapes)}
    assert rec["per_shape_dram_write"] == {f"M{m}": 2500 for m in shapes}     # Kbyte -> bytes
    assert rec["per_shape_us_under_ncu"]["M512"] == 15.0
    expect = np.mean([1_000_000 * (i + 1) + 2500 for i in range(len(shapes))])
    assert rec["dram_bytes_per_launch"] == int(round(expect))
    assert rec["source_hash"] == source_hash()


def test_traffic_summary_rejects_a_wrong_launch_count(tmp_path):
    lines = [HEADER] + ncu_rows(0, "void nvfp4_gemm_kernel<16>(x)", 1, 0, 1.0)
    p = tmp_path / "t.csv"
    p.write_text("".join(lines))
    with pytest.raises(SystemExit):
        profile_case.summarize_traffic(str(p), str(tmp_path / "o.json"), iters=2)


def test_binding_rejects_mismatched_k_before_any_call():
    import nvfp4_block_scaled_gemm_b200 as nv
    A = torch.zeros((4, 64), dtype=torch.uint8)          # K = 128
    sA = torch.zeros((4, 8), dtype=torch.uint8)
    with pytest.raises(ValueError, match="K mismatch"):
        nv.gemm(A, sA, torch.zeros((8, 32), dtype=torch.uint8), torch.zeros((8, 4), dtype=torch.uint8), 1.0)
    with pytest.raises(ValueError, match="K mismatch"):
        nv.gemm_sparse24(A, sA, torch.zeros((8, 16), dtype=torch.uint8), torch.zeros((8, 4), dtype=torch.uint8),
                         torch.zeros((8, 4), dtype=torch.uint8), 1.0)
    with pytest.raises((ValueError, TypeError)):     # metadata of the wrong width
        nv.gemm_sparse24(A, sA, torch.zeros((8, 32), dtype=torch.uint8), torch.zeros((8, 4), dtype=torch.uint8),
                         torch.zeros((8, 8), dtype=torch.uint8), 1.0)
