"""bench.py's host-side bookkeeping, on the CPU: which kernel does each
workload's pair work, how pairs, kernel evaluations and tensor-core FLOPs are
counted per step, and when the committed ncu traffic figure may be reported."""
import hashlib
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402


def test_dominant_kernel_of_each_workload():
    want = {"d3_10k": "sd_kernel", "d3_100k": "sd_kernel", "d3_1m_lse": "sd_kernel",
            "d32_c32": "tc_gauss_kernel", "d32_c1_bwd": "tc_gauss_kernel",
            "b64_d32_f16": "tc_gauss_kernel", "b64_d32_f32": "tc_f32_kernel",
            "b64_d128_f32": "tc_f32_kernel", "d32_c32_f32": "tc_f32_kernel"}
    assert set(want) == set(synth.BY_NAME)
    for name, kernel in want.items():
        k, src = bench.dominant(synth.BY_NAME[name])
        assert k == kernel
        assert os.path.exists(os.path.join(ROOT, "pairwise_reductions_b200", "csrc", src))


def test_pairs_and_kernel_evaluations_per_step():
    w = synth.BY_NAME
    # one output, one pass
    assert bench.pairs_per_step(w["d3_100k"]) == bench.kernel_evals_per_step(w["d3_100k"]) == 10 ** 10
    # the sum and the log-sum-exp: two outputs, two passes
    assert bench.pairs_per_step(w["d3_1m_lse"]) == 2 * 10 ** 12
    assert bench.kernel_evals_per_step(w["d3_1m_lse"]) == 2 * 10 ** 12
    # forward + backward: the pairs once; one sweep of exponentials in one call
    # (fp16, C = 1, D = 32), two for the two-call path
    p = 4 * 16384 * 16384
    assert bench.pairs_per_step(w["d32_c1_bwd"]) == p
    assert bench.fused_fwd_bwd(w["d32_c1_bwd"])
    assert bench.kernel_evals_per_step(w["d32_c1_bwd"]) == p
    assert bench.kernel_evals_per_step(w["d32_c1_bwd"], two_call=True) == 2 * p


def test_tensor_flops_per_step():
    w = synth.BY_NAME
    per = lambda n: bench.tensor_flops_per_step(w[n]) / w[n].pairs
    # CUDA-core path (fp32, D <= 8) and the mixed-pass backward: no tensor roofline
    assert per("d3_100k") == per("d3_1m_lse") == per("d32_c1_bwd") == 0
    # fp32, D > 8: three fp16-part products per value product (one register
    # channel: the similarity alone; 32 channels: P.v on the tensor cores too)
    assert per("b64_d32_f32") == 3 * 2 * 32
    assert per("b64_d128_f32") == 3 * 2 * 128
    assert per("d32_c32_f32") == 3 * 2 * 32 + 3 * 2 * 32
    # fp16: rows augmented by the two norm terms; one channel summed in registers
    assert per("b64_d32_f16") == 2 * (32 + 2)
    assert per("d32_c32") == 2 * (32 + 2) + 2 * 32


def test_traffic_figure_only_while_the_kernel_source_is_unchanged(tmp_path, monkeypatch):
    lines = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "traffic.txt"))
             if ln.strip() and not ln.startswith("#")]
    assert lines, "no traffic lines"
    for f in lines:
        assert len(f) == 6 and f[1] in synth.BY_NAME and int(f[2]) > 0 and int(f[3]) >= 0
    # a copy of the tree whose source of the first line's kernel differs by one comment
    kernel, wl, rd, wr, src, _ = lines[0]
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    (root / "pairwise_reductions_b200" / "csrc").mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "profiles", "traffic.txt"), root / "profiles" / "traffic.txt")
    shutil.copy(os.path.join(ROOT, "pairwise_reductions_b200", "csrc", src),
                root / "pairwise_reductions_b200" / "csrc" / src)
    monkeypatch.setattr(bench, "ROOT", str(root))
    got, k = bench.traffic_per_launch(synth.BY_NAME[wl])
    assert k == kernel
    sha = hashlib.sha256(open(root / "pairwise_reductions_b200" / "csrc" / src, "rb").read()).hexdigest()
    if sha.startswith(lines[0][5]):
        assert got == int(rd) + int(wr)
    else:
        assert got is None
    with open(root / "pairwise_reductions_b200" / "csrc" / src, "a") as fh:
        fh.write("\n// changed\n")
    assert bench.traffic_per_launch(synth.BY_NAME[wl])[0] is None
