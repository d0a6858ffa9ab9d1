"""Host-side logic of bench.py that the JSON line depends on (CPU).

- The algorithmic work per kernel (the numerators of the roofline fractions)
  follows the formulas stated for each kernel: GEMM flops 2*M*N*K, attention
  bytes 2*4*M*H (+ 4 bytes of valid length per sequence), LayerNorm bytes
  2*2*M*H, residual reads added to the GEMMs that take one.
- The DRAM traffic figure is taken from profiles/traffic.md only while the
  kernel's sources are the ones it was measured on.
- Named workloads have the shapes of the configurations they stand for.
- The per-step statistics are the median and the 10th / 90th percentiles.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import encoder_inputs as EI  # noqa: E402


def test_kernel_work_formulas_bert_base_seq128():
    wl = bench.parse_workload("bert-base:256:128")
    M, H, F, S = 256 * 128, 768, 3072, 128
    w = bench.kernel_work(wl)
    assert w["qkv_gemm"][0] == 2 * M * H * 3 * H
    assert w["qkv_gemm"][1] == 2 * (M * H + H * 3 * H + M * 3 * H)
    assert w["out_proj_gemm"][0] == 2 * M * H * H
    assert w["out_proj_gemm"][1] == 2 * (M * H + H * H + M * H) + 2 * M * H     # + residual
    assert w["ffn1_gemm"][0] == 2 * M * H * F
    assert w["ffn2_ln_gemm"][0] == 2 * M * F * H
    assert w["ffn2_ln_gemm"][1] == 2 * (M * F + F * H + M * H) + 2 * M * H
    assert w["attention"] == (4 * M * S * H, 2 * 4 * M * H + 4 * 256)
    assert w["ln1"] == (0.0, 2 * 2 * M * H)
    # Dense GEMM flops per token per layer 2H(3H + H + 2F): 14.16 MFLOP for BERT-Base.
    per_token = sum(w[k][0] for k in ("qkv_gemm", "out_proj_gemm", "ffn1_gemm", "ffn2_gemm")) / M
    assert per_token == 2 * H * (3 * H + H + 2 * F)
    assert abs(per_token / 1e6 - 14.16) < 0.01


def test_kernel_work_fp32_counts_four_byte_elements():
    wl = bench.parse_workload("tiny-fp32:1")
    M, H = 32, 128
    assert bench.kernel_work(wl)["ln1"] == (0.0, 4 * 2 * M * H)


def test_step_stats_are_median_and_deciles():
    st = bench.step_stats([float(v) for v in (11, 1, 5, 3, 9, 7, 2, 4, 6, 8, 10)])
    assert st == {"median": 6.0, "p10": 2.0, "p90": 10.0}
    st = bench.step_stats([2.0, 1.0])                 # linear interpolation between ranks
    assert st["median"] == pytest.approx(1.5) and st["p10"] == pytest.approx(1.1)


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(512, 1, 2.0) == pytest.approx(256000.0)
    assert bench.job_throughput(512, 4, 2.0) == pytest.approx(4 * 256000.0)


@pytest.mark.parametrize("spec,shape,layers,seq,batch", [
    ("bert-base-s32:512", (12, 64, 3072), 12, 32, 512),
    ("pruned-s32:1024", (4, 32, 512), 12, 32, 1024),
    ("bert-base:256:128", (12, 64, 3072), 12, 128, 256),
    ("bert-base:64:96", (12, 64, 3072), 12, 96, 64),
    ("bert-large:32:512", (16, 64, 4096), 24, 512, 32),
    ("tiny-fp32:1", (4, 32, 512), 1, 32, 1),
])
def test_named_workloads_have_the_config_shapes(spec, shape, layers, seq, batch):
    wl = bench.parse_workload(spec)
    sh = wl.shape
    assert (sh.head_num, sh.size_per_head, sh.ffn_dim) == shape
    assert sh.num_layers == layers and wl.seq == seq and wl.batch == batch
    assert wl.dtype == ("fp32" if spec.startswith("tiny") else "fp16")


def _write_table(path, kernel, workload, nbytes, digest):
    with open(path, "w") as f:
        f.write("| kernel | workload | bytes per launch | source digest | capture |\n|---|---|---:|---|---|\n")
        f.write(f"| {kernel} | {workload} | {nbytes:,} | `{digest}` | x.md |\n")


def test_traffic_is_reported_only_for_the_measured_sources(tmp_path, monkeypatch):
    kernel, workload = "ffn2_ln_gemm", "bert-base-12L-h768-s32-b512-fp16"
    digest = bench.source_digest(kernel)
    assert len(digest) == 16
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # source_digest reads the sources under ROOT: keep reading the real ones.
    monkeypatch.setattr(bench, "source_digest", lambda k: digest)
    table = tmp_path / "profiles" / "traffic.md"
    _write_table(table, kernel, workload, 142873856, digest)
    assert bench.measured_traffic(kernel, workload) == 142873856.0
    assert bench.measured_traffic(kernel, "another-workload") is None
    assert bench.measured_traffic("qkv_gemm", workload) is None
    _write_table(table, kernel, workload, 142873856, "0" * 16)         # sources changed since
    assert bench.measured_traffic(kernel, workload) is None


def test_source_digest_depends_on_every_listed_file():
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "transformer_encoder_bert_b200", "csrc", f)), (kernel, f)
    assert bench.source_digest("ln1") != bench.source_digest("qkv_gemm")
    assert bench.source_digest("qkv_gemm") == bench.source_digest("ffn1_gemm")    # same sources


def test_kernel_names_follow_launch_order():
    assert bench.kernel_names(7 * 2, 2, False) == bench.KERNEL_NAMES * 2
    assert bench.kernel_names(6 * 12, 12, False) == bench.KERNEL_NAMES_FFN2_LN * 12
    assert bench.kernel_names(6 * 12, 12, False, ffn2_ln_off=True) == bench.KERNEL_NAMES_OPROJ_LN * 12
    assert bench.kernel_names(5 * 12, 12, False) == bench.KERNEL_NAMES_FUSED * 12
    names = bench.kernel_names(6 * 12 + 3, 12, True)
    assert names[:2] == ["offsets", "pack"] and names[-1] == "unpack" and len(names) == 75


def test_roofline_divides_by_the_burst_tensor_peak():
    """The GEMMs run for microseconds inside millisecond steps: the clock-burst
    matmul peak is the denominator, and the fraction recomputes from the line."""
    wl = bench.parse_workload("bert-base-s32:512")
    peaks = {"hbm_gbs": 6558.4, "bf16_tflops": 1653.4, "bf16_tflops_sustained": 1397.7}
    per_kernel = {k: [0.1, 0.1] for k in bench.KERNEL_NAMES_FFN2_LN}
    per_kernel["ffn2_ln_gemm"] = [0.0736, 0.0736]
    kernels, work = bench.kernel_table(wl, None, per_kernel, peaks, packed=False)
    roof = bench.roofline_of(kernels, work, "ffn2_ln_gemm", peaks, "measured", None)
    assert roof["peak"] == 1653.4
    assert roof["achieved"] == pytest.approx(2 * 16384 * 3072 * 768 / 73.6e-6 / 1e12)
    # in-graph time: the kernel's share of the traced forward times the graph step,
    # per launch (two traced forwards of one launch each per kernel here)
    kg, _ = bench.kernel_table(wl, None, per_kernel, peaks, packed=False, graph_ms=0.5, forwards=2)
    share = 0.0736 / (0.0736 + 5 * 0.1)
    assert kg["ffn2_ln_gemm"]["graph_us"] == pytest.approx(share * 0.5 * 1e3)
    rg = bench.roofline_of(kg, work, "ffn2_ln_gemm", peaks, "measured", None)
    assert rg["achieved"] == pytest.approx(2 * 16384 * 3072 * 768 / (share * 0.5e-3) / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1653.4)
    ln = bench.roofline_of(kernels, work, "ln1", peaks, "measured", None)
    assert ln["bound"] == "hbm" and ln["frac"] == pytest.approx(2 * 2 * 16384 * 768 / 0.1e-3 / 1e9 / 6558.4)


def test_decoder_workload_and_flops():
    wl = bench.decoder_workload("decoder-base:8:64:128")
    assert (wl.batch, wl.tgt_seq, wl.mem_seq, wl.shape.num_layers) == (8, 64, 128, 12)
    H, F = 768, 3072
    mt, ms = 8 * 64, 8 * 128
    gemm = 2 * mt * H * (6 * H + 2 * F) + 2 * ms * H * 2 * H
    attn = 4 * mt * 64 * H / 2 + 4 * mt * 128 * H
    assert bench.decoder_flops(wl) == pytest.approx(12 * (gemm + attn))
