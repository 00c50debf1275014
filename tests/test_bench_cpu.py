"""Host logic of bench.py that needs no GPU: the kernel the launcher picks per
workload, the algorithmic bytes and flops, and the reading of the committed ncu
summaries (a summary counts only while the kernel's code is the one it describes)."""
import importlib.util
import os
import shutil

import pytest

from gated_delta_rule_102_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_kernel_choice_per_workload():
    b = _bench()
    w = synth.WORKLOADS
    assert b.kernel_for(w["batch64"], 148) == "decode_ws_kernel"
    assert b.kernel_for(w["pool384_batch256"], 148) == "decode_ws_kernel"
    assert b.kernel_for(w["single_seq"], 148) == "decode_fused_tma_kernel"
    assert b.kernel_for(w["tiny_d16"], 148) == "decode_fused_tma_kernel"
    # several tokens per sequence: the chunked tensor-core kernel at dk = dv = 128, else the
    # register-tile kernel
    assert b.kernel_for(w["multitoken_b32_t16"], 148) == "decode_chunk_kernel"
    assert b.kernel_for(w["ragged_b64_t16"], 148) == "decode_chunk_kernel"
    assert b.kernel_for(w["multitoken_b32_t16"].replace(head_v_dim=64), 148) == "decode_mt_kernel"


def test_algorithmic_bytes_and_flops_match_the_stated_counts():
    b = _bench()
    w = synth.WORKLOADS
    # per sequence per single-token step 4,325,508 B, per launch 66,048 B of weights
    assert b.algorithmic_bytes(w["batch64"]) == 64 * 4325508 + 66048 == 276898560
    assert b.algorithmic_bytes(w["pool384_batch256"]) == 256 * 4325508 + 66048
    # 7 flops per state element per token: 1.879 GFLOP per multi-token launch
    assert b.algorithmic_flops(w["multitoken_b32_t16"]) == 7 * 32 * 16 * 32 * 128 * 128 == 1879048192
    # a ragged launch whose sequences all bring T tokens moves what the uniform one moves,
    # plus its B+1 offsets; sequences without tokens move nothing
    import numpy as np
    wu = w["multitoken_b32_t16"]
    nb, nf = b.ragged_bytes_flops(wu, np.full(32, 16))
    assert nb == b.algorithmic_bytes(wu) + 33 * 4 and nf == b.algorithmic_flops(wu)
    nb0, nf0 = b.ragged_bytes_flops(wu, np.r_[np.full(16, 16), np.zeros(16, int)])
    assert nf0 == nf // 2 and nb0 == nb - 16 * (nb - b.ragged_bytes_flops(wu, np.zeros(32, int))[0]) // 32


def test_profile_counts_only_for_the_code_it_was_taken_on(tmp_path, monkeypatch):
    b = _bench()
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "gated_delta_rule_102_b200", "csrc"), root / "gated_delta_rule_102_b200" / "csrc")
    shutil.copytree(os.path.join(ROOT, "include"), root / "include")
    (root / "profiles").mkdir()
    for kernel, wl in (("decode_ws_kernel", "batch64"), ("decode_mt_kernel", "multitoken_b32_t16")):
        # a summary in the committed format, stamped with the code as it is now
        (root / "profiles" / f"{kernel}_{wl}.md").write_text(
            f"# {kernel}\n\nkernel source hash: `{{h}}`\n\n| quantity | value |\n|---|---|\n"
            f"| dram bytes per launch: | 123456789 |\n")
    monkeypatch.setattr(b, "ROOT", str(root))
    for kernel, wl in (("decode_ws_kernel", "batch64"), ("decode_mt_kernel", "multitoken_b32_t16")):
        f = root / "profiles" / f"{kernel}_{wl}.md"
        f.write_text(f.read_text().replace("{h}", b.kernel_source_hash(kernel)))
    assert b.profiled_traffic("decode_ws_kernel", "batch64") == 123456789
    f = root / "gated_delta_rule_102_b200" / "csrc" / "gdn_decode_persistent.cu"
    f.write_text(f.read_text() + "\n// a comment changes nothing\n")
    assert b.profiled_traffic("decode_ws_kernel", "batch64") is not None
    f.write_text(f.read_text() + "\nstatic int extra_code = 1;\n")
    assert b.profiled_traffic("decode_ws_kernel", "batch64") is None
    # the other kernel's summary is unaffected
    assert b.profiled_traffic("decode_mt_kernel", "multitoken_b32_t16") is not None
