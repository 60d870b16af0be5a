"""The work figures bench.py divides by (host-side arithmetic, no GPU).

The roofline fractions the bench reports are algorithmic work / measured time /
measured peak, so the work must be right. These tests re-derive it another way:
FLOPs per token and head from the matrix shapes of each GEMM phase, the
aggregation's bytes chunk by chunk, and the whole call's compulsory bytes from
its inputs and outputs, and check the recorded ncu traffic is only used for the
kernel sources it was taken on.
"""
import os
import shutil

import pytest

import e2ttt_inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def gemm_flops(m, n, k):
    return 2 * m * n * k


def test_forward_flops_from_gemm_shapes(bench):
    """Per chunk of C tokens and one head: G1 multiplies the 2C query and key rows
    by the hidden weights, G2 the 2C activation rows by W2, G3 the C residual rows
    by W2, G4 forms two weighted sums (a and b) for every state matrix."""
    for name in ("layer_1p3b_2k", "swiglu_d128", "layer_1p3b_2k_gelu", "tiny_linear"):
        w = gen.BY_NAME[name]
        C, dk, dv, dh = w.C, w.d_k, w.d_v, w.d_h
        if w.kind == gen.LINEAR:
            ref = gemm_flops(2 * C, dv, dk) + 2 * gemm_flops(dv, dk, C)
        else:
            nf = 2 if w.kind == gen.SWIGLU else 1
            ref = (gemm_flops(2 * C, nf * dh, dk) + gemm_flops(2 * C, dv, dh) + gemm_flops(C, dh, dv)
                   + 2 * (gemm_flops(nf * dh, dk, C) + gemm_flops(dv, dh, C)))
        got = sum(bench.phase_flops_per_token_head(w).values()) * C
        assert got == ref, (name, got, ref)
    w = gen.BY_NAME["layer_1p3b_2k"]
    assert bench.fwd_flops(w) == 26 * w.d_k * w.d_h * w.B * w.H * w.T
    g = gen.BY_NAME["layer_1p3b_2k_gelu"]
    assert bench.fwd_flops(g) == 18 * g.d_k * g.d_h * g.B * g.H * g.T


def test_backward_flops(bench):
    """The tensor-core backward's launches: 52 d d_h of adjoint work per token and
    head plus 14 of recomputation (R1 8, R2 2, du 2 in R3 and 2 more in E5, whose
    second accumulator forms it again), or 10 with the forward's E and dH saved;
    training counts the forward and the 52 (twice the forward's 26)."""
    f = bench.TC_BWD_FLOPS
    recompute = ("tcb_r1_h", "tcb_r2_e", "tcb_r3_q1", "tcb_d1_d2", "tcb_e3_dk1", "tcb_e4_eb",
                 "tcb_e5_hb", "tcb_dk2_dq", "tcb_dw")
    saved = ("tcb_r1_h", "tcb_q1_hbq", "tcb_d1_d2", "tcb_e3_dk1", "tcb_e4_eb", "tcb_e5_hb",
             "tcb_dk2_dq", "tcb_dw")
    # one chunk's launches: 52 of adjoint plus the recomputed H (8), E (2), du
    # (2, in R3) and du again (2, in E5); with saved E and dH only H and E5's du
    assert sum(f[n] for n in recompute) == 52 + 14
    assert sum(f[n] for n in saved) == 52 + 10
    assert f["tcb_r3_q1"] == f["tcb_q1_hbq"] + 2
    w = gen.BY_NAME["train_1p3b_2k"]
    assert bench.train_flops(w) == 78 * w.d_k * w.d_h * w.B * w.H * w.T


def test_aggregation_bytes_chunk_by_chunk(bench):
    """G4 of the 1.3B layer, one launch averaged over the step's chunks: bf16
    operands (dH, aK, bK, aE, bE, A_k) read once per chunk; the fp32 state read
    once (W0 only in the first chunk, W and M after), W and M written every chunk
    and the bf16 copy of W written for every chunk but the last."""
    w = gen.BY_NAME["layer_1p3b_2k"]
    BH, C, NC = w.B * w.H, w.C, w.T // w.C
    dk, dv, dh = w.d_k, w.d_v, w.d_h
    S = 2 * dh * dk + dv * dh
    operands = 2 * (2 * C * dh + 2 * C * dk + 2 * C * dv + C * dh)   # dH, aK, bK, aE, bE, A_k (bf16)
    total = 0
    for ci in range(NC):
        reads = S * 4 if ci == 0 else 2 * S * 4      # M0 = 0 is not read
        writes = 2 * S * 4 + (S * 2 if ci + 1 < NC else 0)
        total += operands + reads + writes
    per_launch = total / NC * BH
    got = bench.kernel_work(w, has_m0=False)["tc_g4_aggregate_state"][2]
    assert got == per_launch == 291504128.0


def test_algorithmic_bytes_are_the_calls_compulsory_traffic(bench):
    """The algorithmic bytes charged to the forward's launches add up to the
    call's compulsory traffic less the gates (which K1 reads): q, k with the
    first GEMM phase, v, out with the phase that forms out, W0, M0, W_end, M_end
    once per call with the aggregation; intermediates and the per-chunk state
    round trips are implementation bytes only."""
    w = gen.BY_NAME["layer_1p3b_2k"]
    NC = w.T // w.C
    work = bench.kernel_work(w, has_m0=True)
    per_call = sum(NC * work[n][1] for n in ("tc_g1_h_act", "tc_g2_y_out_e", "tc_g3_da_dh",
                                             "tc_g4_aggregate_state"))
    gates = 12 * w.B * w.H * w.T
    assert per_call == bench.algorithmic_bytes(w) - gates
    assert work["tc_shadow_init"][1] == work["tc_scale_keys"][1] == work["tc_prep"][1] == 0.0
    assert work["tc_prep"][2] == work["tc_shadow_init"][2] + work["tc_scale_keys"][2]
    # implementation bytes never undercount the algorithmic ones
    for n, (f, alg, impl) in work.items():
        assert impl >= alg, n


def test_roofline_bound_follows_the_algorithmic_work(bench):
    """G4 of the 1.3B layer does 12 d d_h FLOPs per token and head and carries a
    quarter of the call's state bytes: at the measured peaks that is
    tensor-bound, and the fraction is FLOPs / time / bf16 peak."""
    w = gen.BY_NAME["layer_1p3b_2k"]
    f, alg, impl = bench.kernel_work(w, has_m0=False)["tc_g4_aggregate_state"]
    assert f == 12 * w.d_k * w.d_h * w.B * w.H * w.C
    peaks = {"hbm_gbs": 6557.4, "bf16_tflops": 1667.1, "source": "measured"}
    r = bench.roofline_of(f, alg, 57.97e-6, peaks)
    assert r["bound"] == "tensor"
    assert abs(r["frac"] - f / 57.97e-6 / 1667.1e12) < 1e-12
    assert 0.26 < r["frac"] < 0.27


def test_call_bytes_match_the_compulsory_traffic(bench):
    """One forward call of the 1.3B layer: q, k, v in and out out (bf16), three
    fp32 gates per token, W0 and M0 in, W_end and M_end out (fp32): about 336 MB."""
    w = gen.BY_NAME["layer_1p3b_2k"]
    toks = w.B * w.H * w.T
    S = 2 * w.d_h * w.d_k + w.d_v * w.d_h
    ref = toks * 2 * (w.d_k + w.d_k + w.d_v + w.d_v) + toks * 3 * 4 + 4 * w.B * w.H * S * 4
    assert bench.algorithmic_bytes(w) == ref
    assert 335e6 < ref < 337e6


def test_recorded_traffic_needs_matching_sources(bench, tmp_path, monkeypatch):
    """A profile's traffic figure is used only while the kernel sources hash to
    the value recorded with it."""
    src = tmp_path / "test_weight_layers_chunk_b200" / "csrc"
    src.mkdir(parents=True)
    for rel in bench.KERNEL_SOURCES["tc_"]:
        shutil.copy(os.path.join(ROOT, rel), tmp_path / rel)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_sha("tc_g4_aggregate_state")
    (tmp_path / "profiles").mkdir()
    prof = tmp_path / "profiles" / "tc_g4_aggregate_state__layer_1p3b_2k.md"
    prof.write_text(f"kernel_source_sha: {sha}\ntraffic_bytes_per_launch: 123456\n")
    assert bench.recorded_traffic("tc_g4_aggregate_state", "layer_1p3b_2k") == 123456.0
    with open(tmp_path / bench.KERNEL_SOURCES["tc_"][-1], "a") as f:
        f.write("\n// changed\n")
    assert bench.recorded_traffic("tc_g4_aggregate_state", "layer_1p3b_2k") is None
    assert bench.recorded_traffic("tc_g4_aggregate_state", "other_workload") is None


def test_persistent_forward_work_is_the_sum_of_its_phases(bench):
    """One launch of the persistent forward runs the four GEMM phases of every
    chunk: its FLOPs are the forward's, its algorithmic bytes the call's
    compulsory traffic less the gates."""
    w = gen.BY_NAME["layer_1p3b_2k"]
    work = bench.kernel_work(w, has_m0=False)
    f, alg, impl = work["tc_fwd_persistent"]
    assert f == bench.fwd_flops(w)
    assert alg == bench.algorithmic_bytes(w) - 12 * w.B * w.H * w.T
    NC = w.T // w.C
    assert impl == NC * sum(work[n][2] for n in ("tc_g1_h_act", "tc_g2_y_out_e", "tc_g3_da_dh",
                                                 "tc_g4_aggregate_state"))
