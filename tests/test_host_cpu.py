"""Host-side logic that needs no GPU: the benchmark's byte and ALU accounting and the
seeded generators' layouts."""
import bench
from selective_scan_sfm_b200 import synth


def test_algorithmic_bytes_fixed_layout():
    # bf16 stage-4 shape: x [B,D,T], dt, z [B,D,L], B, C [B,N,L], y [B,D,L], fp32 params
    B, D, T, N, K = 256, 1280, 49, 16, 4
    L = T + 2
    got = bench.algorithmic_bytes(B, D, T, L, N, K, 2, 2)
    assert got == 2 * (B * D * T + 2 * B * D * L + 2 * B * N * L + B * D * L) + 4 * D * (N + 3 + K)


def test_ragged_bytes_equal_fixed_bytes_for_equal_lengths():
    S, D, T, N, K = 8, 64, 30, 16, 4
    L = T + 2
    fixed = bench.algorithmic_bytes(S, D, T, L, N, K, 2, 2)
    ragged = bench.ragged_algorithmic_bytes(S, D, S * L, N, K, 2, 2, aux=True)
    assert ragged == fixed + 4 * (S + 1)  # plus the offsets


def test_alu_peak_is_the_balanced_split():
    E, F = bench.alu_ops_per_element(16, 4)
    assert (E, F) == (20, 80)
    clk = bench.alu_clk_per_element(16, 4)
    # both pipes equally busy at the optimum, never better than either bound alone
    assert clk >= F / bench.FP32_PER_CLK_SM and clk <= E / bench.MUFU_PER_CLK_SM


def test_ragged_generator_packing():
    lens = synth.ragged_lengths(12, 49, 196, seed=3)
    assert len(lens) == 12 and all(51 <= n <= 198 for n in lens)
    d = synth.make_ragged_inputs(lens, D=8, N=4, dtype="f32", seed=3)
    cu = d["cu_seqlens"].tolist()
    assert cu[0] == 0 and cu[-1] == sum(lens) == d["Ltot"]
    assert all(b - a == n for a, b, n in zip(cu[:-1], cu[1:], lens))
    assert tuple(d["x"].shape) == (8, sum(lens) - 2 * 12)
    assert tuple(d["dt"].shape) == (8, sum(lens)) and tuple(d["Bm"].shape) == (4, sum(lens))
    # the same seed draws the same numbers
    d2 = synth.make_ragged_inputs(lens, D=8, N=4, dtype="f32", seed=3)
    assert all((d[k] == d2[k]).all() for k in ("x", "dt", "z", "Bm", "Cm"))
