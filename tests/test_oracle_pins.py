"""The CPU oracle against what the pages and mathematics fix (no GPU).

Each test runs one check from ``pins.py`` on the real oracle. The checks use
closed forms, invariants, torch SDPA in float64 (a library routine), SciPy's
logsumexp, a pure-Python brute force and the page-cited geometry fixture.
"""

import os

import numpy as np
import pytest

import oracle
from packgen import CONFIGS, make_workload
import pins


def test_latent_geometry_fixture(repo_root):
    path = os.path.join(repo_root, "tests", "golden", "latent_geometry.txt")
    rows = [list(map(int, ln.split())) for ln in open(path) if ln.strip() and not ln.startswith("#")]
    grids = {(r[0], r[1]): (r[4], r[5], r[6]) for r in rows}
    for (ih, iw), (gh, gw, n) in grids.items():
        assert ih // 16 == gh and iw // 16 == gw and gh * gw == n
    # every image grid of the workloads is one of the report's sizes
    used = set()
    for idx in range(2, 6):
        for (f, gh, gw, _t) in CONFIGS[idx]["samples"]:
            used.add((gh, gw))
    assert used <= {(g[0], g[1]) for g in grids.values()}


def test_pack_tiny_closed_form():
    pins.check_pack_tiny_closed_form(oracle.pack_build)


def test_pack_vs_brute():
    pins.check_pack_vs_brute(oracle.pack_build)


def test_pack_edit_frames():
    pins.check_pack_edit_frames(oracle.pack_build)


def test_pack_rejects_invalid():
    with pytest.raises(ValueError):
        oracle.pack_build([(2, 4, 4, 0, 0)], 2)
    with pytest.raises(ValueError):
        oracle.pack_build([(3, 4, 4, 0, 0)], 3)
    with pytest.raises(ValueError):
        oracle.pack_build([(1, 4, 4, -1, 0)], 2)


def test_pack_workload_token_counts():
    # closed forms from the workload descriptions
    assert make_workload(1, with_arrays=False).T == 16 * 16 + 20 + 8 * 32 + 12
    assert make_workload(2, with_arrays=False).T == 16384
    assert make_workload(3, with_arrays=False).T == 2 * 64 * 64 + 256 + 16
    assert make_workload(4, with_arrays=False).T == 2 * (2 * 64 * 64 + 256)
    w5 = make_workload(5, with_arrays=False)
    assert 128 * 128 + 512 + 3 * 4096 + 3 * 128 <= w5.T <= 128 * 128 + 512 + 3 * 4096 + 3 * 512


def test_mod_layout():
    pins.check_mod_layout(oracle.adaln_params)


def test_mod_vs_brute():
    pins.check_mod_vs_brute(oracle.adaln_params)


def test_layernorm_moments():
    pins.check_layernorm_moments(oracle.layer_norm_rows)


def test_adaln_zero_map():
    pins.check_adaln_zero_map(oracle.adaln_params, oracle.adaln_modulate,
                              oracle.layer_norm_rows, oracle.gated_residual)


def test_adaln_vs_brute():
    pins.check_adaln_vs_brute(oracle.adaln_params, oracle.adaln_modulate, oracle.pack_build)


def test_rope_identity_and_norm():
    pins.check_rope_identity_and_norm(oracle.rope_apply)


def test_rope_relative_position():
    pins.check_rope_relative(oracle.rope_apply)


def test_rope_textbook_1d():
    pins.check_rope_textbook_1d(oracle.rope_apply)


def test_rope_3d_layout():
    pins.check_rope_3d_layout(oracle.rope_apply)


def test_rope_vs_brute():
    pins.check_rope_vs_brute(oracle.rope_apply, oracle.pack_build)


def test_attention_vs_sdpa():
    pins.check_attention_vs_sdpa(oracle.varlen_attention)


def test_attention_lse():
    pins.check_attention_lse(oracle.varlen_attention)


def test_attention_permutation():
    pins.check_attention_permutation(oracle.varlen_attention)


def test_attention_equal_v():
    pins.check_attention_equal_v(oracle.varlen_attention)


def test_attention_vs_brute():
    pins.check_attention_vs_brute(oracle.varlen_attention)


def test_attention_rows_subset():
    pins.check_attention_rows_subset(oracle.varlen_attention)


def test_gate():
    pins.check_gate(oracle.gated_residual, oracle.adaln_params, oracle.pack_build)


def test_block_rows_subset_matches_full():
    w = make_workload(1)
    p = oracle.pack_build(w.descs, w.rope_axes)
    mod = oracle.adaln_params(w.c, w.W, w.hid)
    full = oracle.block_fwd(w.f32("x"), w.f32("q"), w.f32("k"), w.f32("v"), mod, p, w.rope_axes)
    rows = np.array([0, 100, 275, 276, 543])
    part = oracle.block_fwd(w.f32("x"), w.f32("q"), w.f32("k"), w.f32("v"), mod, p, w.rope_axes,
                            rows=rows)
    for a, b in zip(full, part):
        assert np.allclose(a[rows], b, rtol=0, atol=1e-13)


def test_useful_flops_closed_form():
    w3 = make_workload(3, with_arrays=False)
    n1, n2 = 64 * 64 + 256, 64 * 64 + 16
    assert oracle.useful_attention_flops(w3.descs, 24, 128) == 4 * 128 * 24 * (n1 * n1 + n2 * n2)
    w2 = make_workload(2, with_arrays=False)
    assert w2.descs[-1].is_dummy == 1
    real = sum((d.frames * d.grid_h * d.grid_w + d.n_text) ** 2 for d in w2.descs[:-1])
    assert oracle.useful_attention_flops(w2.descs, 24, 128) == 4 * 128 * 24 * real


def test_cfg_special_weights():
    pins.check_cfg_special_weights(oracle.cfg_combine)


def test_cfg_row_map():
    pins.check_cfg_row_map(oracle.cfg_combine)


def test_cfg_pack_order():
    pins.check_cfg_pack_order(oracle.cfg_combine)


def test_cfg_rejects_mismatched_grids():
    import pytest as _pt
    with _pt.raises(ValueError):
        oracle.cfg_combine(np.zeros((17 + 7 + 14 + 5 + 10, 2)), pins._CFG_DESCS, [(0, 3)], 1.0)


def test_linear_vs_brute():
    pins.check_linear_vs_brute(oracle.modality_linear)


def test_linear_routing():
    pins.check_linear_routing(oracle.modality_linear)


def test_linear_modality_ids_match_pack_build():
    w, tm, _x, _W = pins._linear_case()
    assert np.array_equal(tm, oracle.pack_build(w.descs, 2)["tok_mod"])


def test_gelu():
    pins.check_gelu(oracle.gelu_tanh)


def test_linear_gelu():
    pins.check_linear_gelu(oracle.modality_linear, oracle.gelu_tanh)


def test_mmdit_vs_brute():
    pins.check_mmdit_vs_brute(oracle.mmdit_block_fwd, oracle.pack_build)


def test_mmdit_zero_branches():
    pins.check_mmdit_zero_branches(oracle.mmdit_block_fwd, oracle.pack_build)


def test_mmdit_reduces_to_path():
    pins.check_mmdit_reduces_to_path(oracle.mmdit_block_fwd, oracle.block_fwd,
                                     oracle.adaln_modulate, oracle.pack_build)


def test_mmdit_branch_gates():
    pins.check_mmdit_branch_gates(oracle.mmdit_block_fwd, oracle.pack_build)


def test_mmdit_rows_subset():
    w, ws, mods = pins._mmdit_case(seed=74)
    p = oracle.pack_build(w.descs, 2)
    x = w.f32("x")
    full = oracle.mmdit_block_fwd(x, **ws, **mods, pack=p, H=w.H, D=w.D, rope_axes=2)
    rows = np.array([0, 5, 7, 13])
    part = oracle.mmdit_block_fwd(x, **ws, **mods, pack=p, H=w.H, D=w.D, rope_axes=2, rows=rows)
    assert np.array_equal(full[rows], part)


def test_attention_bwd_vs_autograd():
    pins.check_attention_bwd_vs_autograd(oracle.varlen_attention_bwd)


def test_attention_bwd_finite_diff():
    pins.check_attention_bwd_finite_diff(oracle.varlen_attention_bwd, oracle.varlen_attention)


def test_block_bwd_finite_diff():
    pins.check_block_bwd_finite_diff(oracle.block_bwd, oracle.block_fwd)


def test_adaln_bwd_vs_torch_layer_norm():
    pins.check_adaln_bwd_vs_torch_layer_norm(oracle.adaln_modulate_bwd)


def test_adaln_bwd_invariants():
    pins.check_adaln_bwd_invariants(oracle.adaln_modulate_bwd)


def test_rope_bwd_adjoint():
    pins.check_rope_bwd_adjoint(oracle.rope_bwd, oracle.rope_apply)


def test_adaln_params_bwd_adjoint():
    pins.check_adaln_params_bwd_adjoint(oracle.adaln_params_bwd, oracle.adaln_params)


def test_gelu_bwd_vs_torch():
    pins.check_gelu_bwd_vs_torch(oracle.gelu_tanh_bwd)


def test_linear_bwd_vs_autograd():
    pins.check_linear_bwd_vs_autograd(oracle.modality_linear_bwd)


def test_mmdit_bwd_finite_diff():
    pins.check_mmdit_bwd_finite_diff(oracle.mmdit_block_bwd, oracle.mmdit_block_fwd)


def test_attention_bwd_vs_brute():
    pins.check_attention_bwd_vs_brute(oracle.varlen_attention_bwd)
