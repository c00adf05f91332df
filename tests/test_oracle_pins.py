"""Pins for the CPU oracle: each test ties the oracle to something other than
itself -- a value the pages print, a closed form, an invariant, brute force,
or an independent library routine.  CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from semi_structured_sparse_02_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(values):
    return inputs.to_bf16_bits(np.asarray(values, dtype=np.float32))


# ---------------------------------------------------------------------------
# prune: worked example, brute force over ties, torch top-k recipe
# ---------------------------------------------------------------------------

def test_worked_example_from_the_page():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    v = bf16(g["dense"])
    nib, i0, i1 = orc.prune_group(v)
    assert [i0, i1] == g["kept_indices"]
    assert nib == (i0 | (i1 << 2)) == 0xC
    # the canonical byte holds two groups: pad the row with an all-zero group
    row = np.concatenate([v, bf16([0.0] * 4)]).reshape(1, 8)
    pruned, values, meta = orc.prune_compress_bf16(row)
    assert pruned[0, :4].tolist() == bf16(g["pruned"]).tolist()
    assert values[0, :2].tolist() == bf16([g["dense"][0], g["dense"][3]]).tolist()
    assert meta.tolist() == [[0x4C]]  # group 0 -> low nibble 0xC; zero group keeps 0,1


def _stable_sort_rule(mags):
    # The rule written a second way: sort positions by descending magnitude,
    # equal magnitudes keeping ascending position order; keep the first two.
    order = sorted(range(4), key=lambda i: (-mags[i], i))
    return sorted(order[:2])


def test_prune_brute_force_all_tie_patterns_and_signs():
    levels = [0.0, 1.0, 2.0, 3.0]
    for mags in itertools.product(range(4), repeat=4):
        for signs in itertools.product([1.0, -1.0], repeat=4):
            vals = [s * levels[m] for s, m in zip(signs, mags)]
            _, i0, i1 = orc.prune_group(bf16(vals))
            assert [i0, i1] == _stable_sort_rule([levels[m] for m in mags]), (vals, i0, i1)


def test_prune_agrees_with_torch_topk_recipe_on_tie_free_data():
    # "2:4 Structured Sparsity Explained", section "Running a 2:4 model in
    # PyTorch": keep the top-2 |w| of each group of four via topk.
    W = inputs.normal_bf16((64, 512), 1.0, seed=11)
    w = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).float()
    groups = w.abs().reshape(-1, 4)
    tie_free = torch.tensor([len(set(g.tolist())) == 4 for g in groups])
    mask = torch.zeros_like(groups, dtype=torch.bool)
    mask.scatter_(1, groups.topk(2, dim=1).indices, True)
    pruned, _, _ = orc.prune_compress_bf16(W)
    ours = (torch.from_numpy(pruned.view(np.int16)).view(torch.bfloat16).float()
            .reshape(-1, 4) != 0)
    assert tie_free.float().mean() > 0.95
    assert torch.equal(ours[tie_free], mask[tie_free])


def test_pattern_exactly_two_indices_and_half_zeros():
    W = inputs.normal_bf16((128, 1024), 0.02, seed=3)
    pruned, values, meta = orc.prune_compress_bf16(W)
    nibs = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(128, -1)
    i0, i1 = nibs & 3, nibs >> 2
    assert np.all(i0 < i1)  # two distinct positions per group, ascending
    nz = (pruned.reshape(128, -1, 4) & 0x7FFF) != 0
    assert np.all(nz.sum(-1) <= 2)
    if np.all((W & 0x7FFF) != 0):  # continuous draws: no exact zeros
        assert (pruned & 0x7FFF == 0).mean() == 0.5


def test_kept_zeros_when_group_has_fewer_than_two_nonzeros():
    v = bf16([0.0, 0.0, -0.0, 0.0])
    assert orc.prune_group(v)[1:] == (0, 1)
    v = bf16([0.0, 0.0, 5.0, 0.0])
    assert orc.prune_group(v)[1:] == (0, 2)


# ---------------------------------------------------------------------------
# storage counts
# ---------------------------------------------------------------------------

def test_storage_36_bits_per_4_and_bit_identities():
    s = json.load(open(os.path.join(GOLDEN, "storage.json")))
    X, W = inputs.tiny(0)
    _, values, meta = orc.prune_compress_bf16(W)
    dense_bytes = W.nbytes
    assert values.nbytes + meta.nbytes == 73728
    assert dense_bytes == 131072
    assert (values.nbytes + meta.nbytes) * 64 == dense_bytes * s["fp16_sparse_bits_per_4"]
    assert abs((values.nbytes + meta.nbytes) / dense_bytes - s["fp16_sparse_relative_size_approx"]) < 0.01
    # bits per element of 2:4 on b-bit values = b/2 + 1 (index bits counted)
    bits_per_elem = (values.nbytes + meta.nbytes) * 8 / W.size
    assert bits_per_elem == s["budget_fp16_bits_per_elem"]
    vq, mq, sq, _ = orc.prune_compress_e4m3(W)
    assert (vq.nbytes + mq.nbytes) * 8 / W.size == 5.0  # 0.625 of dense 8-bit
    for m in range(1, 9):  # 2:4 on 2m-bit values costs as much as dense (m+1)-bit
        assert (2 * m) / 2 + 1 == m + 1
    for k in (4, 8, 16):
        assert abs(k / (k / 2 + 1) - 2 * k / (k + 2)) < 1e-12
    assert abs(math.log2(6) / 4 - s["ideal_index_bits_per_elem_approx"]) < 0.005
    # the metadata costs exactly 1 bit per dense element (4 bits per group of 4)
    assert mq.nbytes * 8 / W.size == s["hardware_index_bits_per_elem"]


# ---------------------------------------------------------------------------
# round trip
# ---------------------------------------------------------------------------

def test_decompress_of_compress_is_prune_bit_exact():
    W = inputs.weights_with_outliers(256, 512, seed=5)
    pruned, values, meta = orc.prune_compress_bf16(W)
    assert np.array_equal(orc.decompress(values, meta, 256, 512), pruned)
    vq, mq, sq, _ = orc.prune_compress_e4m3(W)
    assert np.array_equal(mq, meta)  # quantizing does not change which values are kept
    dq = orc.decompress(vq, mq, 256, 512)
    inv = np.array([orc.e4m3_row_scale(float(a))[1] for a in
                    np.abs(orc.bf16_bits_to_f64(W)).max(1).astype(np.float32)], np.float32)
    expect = orc.e4m3_encode(orc.bf16_bits_to_f64(pruned).astype(np.float32) * inv[:, None])
    assert np.array_equal(dq, expect)


# ---------------------------------------------------------------------------
# e4m3
# ---------------------------------------------------------------------------

def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = orc.bf16_bits_to_f64(bits)
    return vals[np.isfinite(vals)]


def test_e4m3_matches_torch_cast_in_range_exhaustive():
    x = _all_finite_bf16()
    for inv in (1.0, 0.37109375, 3.0, 1.0 / 3.0, 1000.0, 1e-3):
        y = (x.astype(np.float32) * np.float32(inv)).astype(np.float32)
        y = y[np.abs(y) < 448.0]
        ours = orc.e4m3_encode(y)
        ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        # torch gives +0 for tiny negatives that round to zero; compare values
        assert np.array_equal(orc.e4m3_decode(ours), orc.e4m3_decode(ref))


def test_e4m3_representables_fixed_points_midpoints_even_saturation():
    codes = [c for c in range(256) if not math.isnan(orc.e4m3_decode(np.array([c]))[0])]
    assert len(codes) == 254
    vals = orc.e4m3_decode(np.array(codes))
    assert np.array_equal(orc.e4m3_encode(vals), np.array(codes, np.uint8)) or \
        np.array_equal(orc.e4m3_decode(orc.e4m3_encode(vals)), vals)
    pos = np.unique(vals[vals >= 0])
    assert pos.max() == 448.0 and pos[1] == 2.0 ** -9
    mids = (pos[:-1] + pos[1:]) / 2
    q = orc.e4m3_decode(orc.e4m3_encode(mids))
    lo_code = orc.e4m3_encode(pos[:-1])
    hi_code = orc.e4m3_encode(pos[1:])
    expect = np.where(lo_code % 2 == 0, pos[:-1], pos[1:])
    assert np.array_equal(q, expect)
    assert np.all(lo_code % 2 != hi_code % 2)
    assert orc.e4m3_encode(np.array([448.0, 460.0, 464.0, 1e4]))[:].tolist() == [0x7E] * 4
    assert orc.e4m3_encode(np.array([-448.0, -1e6])).tolist() == [0xFE, 0xFE]
    grid = np.linspace(-500, 500, 200001).astype(np.float32)
    dec = orc.e4m3_decode(orc.e4m3_encode(grid))
    assert np.all(np.diff(dec) >= 0)


def test_row_scale_closed_form_and_amax_invariant():
    W = inputs.weights_with_outliers(128, 1024, seed=9)
    vq, mq, scales, _ = orc.prune_compress_e4m3(W)
    w = orc.bf16_bits_to_f64(W)
    pruned, _, _ = orc.prune_compress_bf16(W)
    pw = orc.bf16_bits_to_f64(pruned)
    amax = np.abs(w).max(1)
    assert np.array_equal(np.abs(pw).max(1), amax)  # each group keeps its max
    assert np.array_equal(scales, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    # the largest magnitude of each row lands on +-448
    deq = orc.e4m3_decode(vq)
    assert np.all(np.abs(deq).max(1) == 448.0)
    s, inv = orc.e4m3_row_scale(0.0)
    assert (s, inv) == (1.0, 0.0)
    q, sc = orc.quantize_rows_e4m3(np.zeros((2, 64), np.uint16))
    assert np.all(q == 0) and np.all(sc == 1.0)


def test_quantized_error_within_half_ulp_of_scaled_value():
    X = inputs.normal_bf16((8, 512), 1.0, seed=21)
    q, s = orc.quantize_rows_e4m3(X)
    x = orc.bf16_bits_to_f64(X)
    deq = orc.e4m3_decode(q) * s[:, None].astype(np.float64)
    # relative spacing of e4m3 normals is 2^-3: error <= half a spacing of |x|
    # plus the subnormal step (2^-9 * s) for tiny values
    bound = np.abs(x) * 2.0 ** -4 * (1 + 1e-6) + 2.0 ** -10 * s[:, None]
    assert np.all(np.abs(deq - x) <= bound)


# ---------------------------------------------------------------------------
# metadata image layout
# ---------------------------------------------------------------------------

def _image_positions(is_8bit):
    rows, K = 128, 128
    pos = {}
    base = np.full((rows, K // 8), 0x44, np.uint8)
    for r in range(rows):
        for g in range(32):
            c = base.copy()
            b = c[r, g // 2]
            c[r, g // 2] = (b & 0xF0) | 0x9 if g % 2 == 0 else (b & 0x0F) | 0x90
            img = orc.meta_image(c, rows, K, is_8bit)
            nibs = np.stack([img & 0xF, img >> 4], -1).reshape(-1)
            hit = np.nonzero(nibs == 0x9)[0]
            assert hit.size == 1
            pos[(r, g)] = int(hit[0])
    return pos


@pytest.mark.parametrize("is_8bit", [False, True])
def test_meta_image_is_a_bijection_with_spec_positions(is_8bit):
    pos = _image_positions(is_8bit)
    assert sorted(pos.values()) == list(range(128 * 32))

    def at(L, w, bit):  # nibble index of image row L, word w, bit offset
        return (L * 16 + w * 4) * 2 + bit // 4

    if not is_8bit:
        assert pos[(0, 0)] == at(0, 0, 0)
        assert pos[(8, 0)] == at(0, 0, 16)
        assert pos[(0, 4)] == at(8, 0, 0)
        assert pos[(16, 8)] == at(16, 1, 0)
        assert pos[(9, 31)] == at(9, 3, 28)
        assert pos[(127, 5)] == at(127, 0, 20)
        assert pos[(119, 5)] == at(127, 0, 4)
    else:
        for (r, g), p in pos.items():
            assert p == r * 32 + g


def test_meta_image_pads_rows_with_valid_nibbles():
    W = inputs.normal_bf16((40, 256), 1.0, seed=2)
    _, _, meta = orc.prune_compress_bf16(W)
    img = orc.meta_image(meta, 40, 256, False)
    assert img.size == 2 * 2048
    img8 = orc.meta_image(meta, 40, 256, True).reshape(2, 128, 16)
    assert np.all(img8[:, 40:, :] == 0x44)


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------

def test_gemm_f64_matches_numpy_matmul():
    g = np.random.default_rng(1)
    X = g.normal(size=(7, 96))
    W = g.normal(size=(13, 96))
    Y, A = orc.gemm_f64(X, W)
    assert np.allclose(Y, X @ W.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(A, np.abs(X) @ np.abs(W).T, rtol=1e-12, atol=1e-12)
    ms = np.array([0, 6, 3]); ns = np.array([12, 0, 5])
    ys, as_ = orc.gemm_f64_sampled(X, W, ms, ns)
    assert np.array_equal(ys, Y[ms, ns]) and np.array_equal(as_, A[ms, ns])


def test_sparse_sum_equals_dense_product_of_pruned_matrix_exactly():
    g = np.random.default_rng(2)
    Xi = g.integers(-8, 9, size=(9, 64)).astype(np.float32)
    Wi = g.integers(-8, 9, size=(17, 64)).astype(np.float32)
    Wb = bf16(Wi)
    pruned, values, meta = orc.prune_compress_bf16(Wb)
    Xd = Xi.astype(np.float64)
    Yd, _ = orc.gemm_f64(Xd, orc.bf16_bits_to_f64(pruned))
    Ys = orc.gemm_sparse_f64(Xd, orc.bf16_bits_to_f64(values), meta)
    assert np.array_equal(Yd, Ys)


def test_already_two_four_weights_reduce_to_dense_gemm():
    g = np.random.default_rng(3)
    N, K = 16, 64
    W = np.zeros((N, K), np.float32)
    for n in range(N):
        for q in range(K // 4):
            idx = g.choice(4, size=2, replace=False)
            W[n, 4 * q + idx] = g.integers(1, 9, size=2) * g.choice([-1, 1], size=2)
    Wb = bf16(W)
    pruned, values, meta = orc.prune_compress_bf16(Wb)
    assert np.array_equal(pruned, Wb)  # prune is the identity on 2:4 input
    X = g.integers(-5, 6, size=(5, K)).astype(np.float64)
    Ys = orc.gemm_sparse_f64(X, orc.bf16_bits_to_f64(values), meta)
    assert np.array_equal(Ys, X @ W.astype(np.float64).T)


# ---------------------------------------------------------------------------
# hybrid tiles
# ---------------------------------------------------------------------------

def test_hybrid_dense_tiles_and_sparse_tiles():
    rows, K = 256, 512
    W = inputs.normal_bf16((rows, K), 0.02, seed=4)
    mask = inputs.hybrid_mask(rows, K, seed=4)
    assert mask.sum() == round(0.25 * mask.size)
    vq, mq, sq, dq = orc.prune_compress_e4m3(W, mask)
    vq0, mq0, sq0, _ = orc.prune_compress_e4m3(W)
    q_dense, s_dense = orc.quantize_rows_e4m3(W)
    pruned0 = orc.decompress(vq0, mq0, rows, K)  # the all-sparse matrix in dense form
    assert np.array_equal(sq, sq0) and np.array_equal(sq, s_dense)
    for rb in range(2):
        for kt in range(4):
            rs, ks = slice(128 * rb, 128 * rb + 128), slice(128 * kt, 128 * kt + 128)
            vs = slice(64 * kt, 64 * kt + 64)
            ms_ = slice(16 * kt, 16 * kt + 16)
            if mask[rb, kt]:
                assert np.all(vq[rs, vs] == 0) and np.all(mq[rs, ms_] == 0x44)
                assert np.array_equal(dq[rs, ks], q_dense[rs, ks])
            else:
                assert np.array_equal(vq[rs, vs], vq0[rs, vs])
                assert np.array_equal(mq[rs, ms_], mq0[rs, ms_])
                # a sparse tile appears in the dense image pruned: exactly the
                # round trip of its compressed form, two zero bytes per group
                assert np.array_equal(dq[rs, ks], pruned0[rs, ks])
                assert np.all((dq[rs, ks].reshape(128, 32, 4) == 0).sum(axis=2) >= 2)
    # bf16 output: the dense image is the original at dense tiles and the
    # plain 2:4 prune elsewhere
    vb, mb, db = orc.prune_compress_bf16_hybrid(W, mask)
    pruned_b, _, _ = orc.prune_compress_bf16(W)
    dm = np.kron(mask, np.ones((128, 128), np.uint8)).astype(bool)
    assert np.array_equal(db, np.where(dm, W, pruned_b))


# ---------------------------------------------------------------------------
# tactic rule and manifest arithmetic
# ---------------------------------------------------------------------------

def test_manifest_example_arithmetic_and_tactic_rule():
    m = json.load(open(os.path.join(GOLDEN, "manifest_example.json")))
    assert m["sparse_selected_layers"] + m["dense_fallback_layers"] == m["candidate_layers"]
    assert round(m["sparse_selected_layers"] / m["eligible_layers"], 4) == m["sparse_selection_ratio"]
    assert orc.select_tactic([1.0, 2.0, 3.0], [2.0, 2.0, 2.0])[0] == "dense"   # tie -> dense
    assert orc.select_tactic([1.0, 1.5, 9.0], [2.0, 2.0, 2.0])[0] == "sparse"
    cov = orc.sparse_gpu_time_coverage([("sparse", 0.684), ("dense", 0.316)])
    assert abs(cov - m["sparse_gpu_time_coverage"]) < 1e-12


# ---------------------------------------------------------------------------
# 2:4 energy loss: the page's worked example, closed forms, brute force
# ---------------------------------------------------------------------------

def test_energy_loss_worked_example():
    # the page's group keeps 0.42 and 0.31 and drops -0.18 and 0.07: the
    # dropped share is (0.18^2 + 0.07^2) / (sum of all four squares), here
    # on the bf16 values of the four numbers
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    v = bf16(g["dense"])
    x = [float(t) for t in torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).float()]
    dropped, total, share, tensor = orc.energy_loss(v.reshape(1, 4))
    assert dropped[0] == x[1] ** 2 + x[2] ** 2
    assert total[0] == sum(t * t for t in x)
    assert share[0] == pytest.approx(0.0373 / 0.3098, rel=2e-2)  # the decimal values, before bf16 rounding
    assert tensor == share[0]


def test_energy_loss_closed_forms():
    # equal magnitudes in every group: exactly half the energy is dropped
    row = bf16(np.tile([1.5, -1.5, 1.5, -1.5], 16)).reshape(2, 32)
    _, _, share, tensor = orc.energy_loss(row)
    assert share.tolist() == [0.5, 0.5] and tensor == 0.5
    # two zeros in every group (an already 2:4 tensor): nothing is dropped
    row = bf16(np.tile([0.0, 3.0, 0.0, -2.0], 8)).reshape(1, 32)
    assert orc.energy_loss(row)[2][0] == 0.0
    # a row of zeros has no energy: share 0 (reading)
    assert orc.energy_loss(np.zeros((1, 8), np.uint16))[2][0] == 0.0
    # scaling by a power of two scales both energies alike: the share is unchanged
    W = inputs.normal_bf16((4, 64), 1.0, seed=11)
    W2 = bf16(torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).float().numpy() * 8.0)
    assert np.array_equal(orc.energy_loss(W)[2], orc.energy_loss(W2)[2])


def test_energy_loss_brute_force_by_sorting():
    # independent of the prune rule: in every group the two smallest squares
    # are dropped (ties do not matter for the energy)
    W = inputs.student_t_bf16((6, 128), 3.0, seed=5)
    x = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).double().numpy()
    sq = np.sort((x.reshape(6, 32, 4)) ** 2, axis=2)
    dropped = sq[:, :, :2].sum(axis=(1, 2))
    total = (x ** 2).sum(axis=1)
    d, t, share, tensor = orc.energy_loss(W)
    assert np.allclose(d, dropped, rtol=1e-14, atol=0) and np.allclose(t, total, rtol=1e-14, atol=0)
    assert tensor == pytest.approx(dropped.sum() / total.sum(), rel=1e-14)


# ---------------------------------------------------------------------------
# pairwise 4:8 sparsity with NVFP4 values (the next row after the 2:4 path)
# ---------------------------------------------------------------------------

# E2M1 magnitudes as tabulated in the OCP microscaling specification
E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_table_ties_to_even_and_saturation():
    vals = orc.e2m1_decode(np.arange(16))
    assert list(vals[:8]) == E2M1_MAGNITUDES
    assert list(-vals[8:]) == E2M1_MAGNITUDES and all(np.signbit(vals[8:]))
    # representable values are fixed points
    for c, m in enumerate(E2M1_MAGNITUDES):
        assert orc.e2m1_encode([m])[0] == c
        assert orc.e2m1_encode([-m])[0] == c | 8
    # midpoints go to the neighbour whose code is even (mantissa bit 0)
    mids = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in mids.items():
        assert orc.e2m1_decode(orc.e2m1_encode([x]))[0] == want
        assert orc.e2m1_decode(orc.e2m1_encode([-x]))[0] == -want
    # off-midpoint values go to the nearest; beyond 6 saturates
    for x in (0.26, 0.74, 1.26, 2.49, 2.51, 4.9, 5.1, 6.0, 6.5, 1e6):
        got = orc.e2m1_decode(orc.e2m1_encode([x]))[0]
        near = min(E2M1_MAGNITUDES, key=lambda m: abs(m - min(x, 6.0)))
        assert got == near, (x, got)
    # monotone on a fine grid
    grid = np.linspace(-7, 7, 2801)
    dec = orc.e2m1_decode(orc.e2m1_encode(grid))
    assert np.all(np.diff(dec) >= 0)


def _pair_group(energies_as_values, signs=(1, 1, 1, 1), split=False):
    """Eight bf16 values whose pair j carries the given value (as one element,
    or split over both elements when split)."""
    v = []
    for j, x in enumerate(energies_as_values):
        a = signs[j] * float(x)
        v.extend([0.0, a] if split else [a, 0.0])
    return bf16(np.array(v, np.float32))


def test_pair_rule_brute_force_all_tie_patterns():
    """Every ordering (with ties) of the four pair weights, against the rule
    written as a stable sort: the two heaviest pairs, ties to the lower pair."""
    for pattern in itertools.product(range(4), repeat=4):
        for signs in ((1, 1, 1, 1), (-1, 1, -1, 1)):
            for split in (False, True):
                g = _pair_group(pattern, signs, split)
                nib, p0, p1 = orc.prune_pairs8(g)
                order = sorted(range(4), key=lambda j: (-pattern[j] ** 2, j))
                want = sorted(order[:2])
                assert [p0, p1] == want, (pattern, signs, split)
                assert nib == want[0] | (want[1] << 2)


def test_pair_rule_weighs_energy_not_the_largest_element():
    # pair 0 holds the largest element (3) but less energy (9) than pairs 1
    # and 2 (2.25^2 * 2 = 10.125 each): the energy reading drops it
    g = bf16(np.array([3.0, 0.0, 2.25, 2.25, 2.25, 2.25, 0.5, 0.5], np.float32))
    nib, p0, p1 = orc.prune_pairs8(g)
    assert (p0, p1) == (1, 2)


def test_pairwise_48_keeps_four_aligned_elements():
    W = inputs.normal_bf16((64, 256), 1.0, seed=21)
    P = orc.prune_pairs_bf16(W)
    kept = (P != 0).reshape(64, 32, 4, 2)
    # whole pairs only, two pairs per group of eight
    assert np.all(kept[..., 0] == kept[..., 1])
    assert np.all(kept[..., 0].sum(axis=2) == 2)
    assert np.array_equal(P[P != 0], W[P != 0])


def test_pairwise_48_energy_closed_form_on_gaussian_data():
    """A pair of N(0,1) values has chi-square(2) energy, exponential with mean
    2; dropping the lighter two of four drops 2/4 + (2/4 + 2/3) = 5/3 of the
    group's expected 8, i.e. 5/24.  The pages put pairs at about one and a half
    times the energy that element-wise 2:4 removes from Gaussian data."""
    W = inputs.normal_bf16((2048, 1024), 1.0, seed=22)
    _, _, _, e48 = orc.energy_loss_48(W)
    _, _, _, e24 = orc.energy_loss(W)
    assert abs(e48 - 5.0 / 24.0) < 2e-3
    assert 1.4 < e48 / e24 < 1.7


def test_energy_loss_48_brute_force_by_sorting():
    W = inputs.normal_bf16((8, 64), 1.0, seed=23)
    dropped, total, share, tensor = orc.energy_loss_48(W)
    x = W.view(np.uint16).astype(np.uint32) << 16
    xf = x.view(np.float32).astype(np.float64).reshape(8, 8, 4, 2)
    e = (xf ** 2).sum(axis=3)                            # pair energies [rows, groups, 4]
    drop = np.sort(e, axis=2)[:, :, :2].sum(axis=(1, 2))  # the two lightest pairs per group
    assert np.allclose(dropped, drop, rtol=0, atol=1e-12)
    assert np.allclose(total, (xf ** 2).sum(axis=(1, 2, 3)), rtol=0, atol=1e-12)


def test_nvfp4_scales_closed_forms():
    amax = np.float32(3.75)
    st = orc.nvfp4_tensor_scale(float(amax))
    assert np.float32(st) == amax / np.float32(2688.0)   # 448 * 6
    assert orc.nvfp4_tensor_scale(0.0) == 1.0
    # the tensor's own amax gets the largest block code, 448
    b = orc.nvfp4_block_code(float(amax), st)
    assert orc.e4m3_decode(np.array([b], np.uint8))[0] == 448.0
    # the block's largest value lands on the E2M1 code of 6: the E4M3 scale is
    # off by at most 1/16, so |v| / S stays within [5.6, 6.5]
    g = np.random.default_rng(24)
    for _ in range(200):
        amax_b = np.float32(g.uniform(1e-3, 3.75))
        bb = orc.nvfp4_block_code(float(amax_b), st)
        assert orc.e2m1_decode(np.array([orc.nvfp4_code(float(amax_b), bb, st)]))[0] == 6.0
    assert orc.nvfp4_block_code(0.0, st) == 0 and orc.nvfp4_code(1.0, 0, st) == 0


def test_nvfp4_48_operand_round_trip_and_error_bound():
    rows, K = 32, 256
    W = inputs.normal_bf16((rows, K), 0.02, seed=25)
    vals, meta, scales, st = orc.nvfp4_48_compress(W)
    assert vals.shape == (rows, K // 4) and meta.shape == (rows, K // 16) and scales.shape == (rows, K // 32)
    # metadata: the pair rule's nibbles, even group in the low nibble
    for r in (0, 7, 31):
        for grp in (0, 5, K // 8 - 1):
            nib = orc.prune_pairs8(W[r, 8 * grp:8 * grp + 8])[0]
            assert (meta[r, grp // 2] >> (4 * (grp % 2))) & 0xF == nib
    P = orc.bf16_bits_to_f64(orc.prune_pairs_bf16(W))
    D = orc.nvfp4_48_dequant(vals, meta, scales, st, rows, K)
    assert np.all(D[P == 0] == 0)                        # nothing at the dropped positions
    S = orc.e4m3_decode(scales).astype(np.float64) * st  # effective scale per 32 positions
    Sfull = np.repeat(S, 32, axis=1)
    # E2M1 gaps are at most 2 (between 4 and 6), so the error is at most one scale
    assert np.all(np.abs(D - P) <= Sfull * (1.0 + 1e-12))
    # storage: 4-bit codes for half the positions, a nibble per 8, a byte per 32
    assert (vals.nbytes + meta.nbytes + scales.nbytes) * 8 / (rows * K) == 2.75


def test_dense_nvfp4_costs_4_5_bits_and_bounds_error():
    """Dense NVFP4 (E4M3 scale per 16 elements) costs 4.5 bits per element
    before the per-tensor scale, the figure the pages use for it."""
    rows, K = 16, 128
    W = inputs.normal_bf16((rows, K), 0.02, seed=26)
    codes, scales, st = orc.nvfp4_quantize(W)
    assert (codes.nbytes + scales.nbytes) * 8 / (rows * K) == 4.5
    D = orc.nvfp4_dequant(codes, scales, st, rows, K)
    X = orc.bf16_bits_to_f64(W)
    S = np.repeat(orc.e4m3_decode(scales).astype(np.float64) * st, 16, axis=1)
    assert np.all(np.abs(D - X) <= S * (1.0 + 1e-12))
    # every block's largest magnitude is represented by the E2M1 code of 6
    c = np.stack([codes & 0xF, codes >> 4], axis=2).reshape(rows, K)
    for r in range(rows):
        for blk in range(K // 16):
            i = np.argmax(np.abs(X[r, 16 * blk:16 * blk + 16]))
            assert orc.e2m1_decode(np.array([c[r, 16 * blk + i]]))[0] in (6.0, -6.0)


def test_nvfp4_32_blocks_for_the_sparse_gemms_dense_operand():
    """The dense operand of the sparse block-scaled GEMM carries one scale per
    32 positions of K: 4.25 bits per element, the same codes as 16-element
    blocks wherever both blocks of 16 share the larger block's scale, and
    the same error bound."""
    rows, K = 8, 256
    X = inputs.normal_bf16((rows, K), 1.0, seed=27)
    c32, s32, st = orc.nvfp4_quantize(X, block=32)
    assert s32.shape == (rows, K // 32) and (c32.nbytes + s32.nbytes) * 8 / (rows * K) == 4.25
    D = orc.nvfp4_dequant(c32, s32, st, rows, K, block=32)
    S = np.repeat(orc.e4m3_decode(s32).astype(np.float64) * st, 32, axis=1)
    assert np.all(np.abs(D - orc.bf16_bits_to_f64(X)) <= S * (1.0 + 1e-12))
    # a 32-block's scale equals the 16-block scale of whichever half holds its amax
    c16, s16, st16 = orc.nvfp4_quantize(X, block=16)
    assert st16 == st
    assert np.array_equal(s32, np.maximum(s16[:, 0::2], s16[:, 1::2]))
    # the sparse GEMM in the oracle is the fp64 product of the dequantized operands;
    # with a 4:8 weight whose pruned entries the product never sees
    W = inputs.normal_bf16((16, K), 0.02, seed=28)
    v, m, sw, stw = orc.nvfp4_48_compress(W)
    Wd = orc.nvfp4_48_dequant(v, m, sw, stw, 16, K)
    Y, A = orc.gemm_f64(D, Wd)
    P = orc.prune_pairs_bf16(W) != 0
    Y2 = np.array([[np.sum(D[i][P[j]] * Wd[j][P[j]]) for j in range(16)] for i in range(rows)])
    assert np.allclose(Y, Y2, rtol=1e-12, atol=1e-15)



def test_nvfp4_48_packing_and_kept_value_scales():
    """R16/R17 by hand on one row of 32 positions: the kept values in ascending
    position, two codes per byte (earlier element low), one nibble per group of
    eight, and scales from the kept values only."""
    # heavy pairs (1, 3) in groups 0 and 2, (0, 2) in groups 1 and 3, light
    # pairs elsewhere; then an 8.0 makes pair 0 the heaviest of group 0
    row = np.zeros(32, np.float32)
    for g in range(4):
        kept = (1, 3) if g % 2 == 0 else (0, 2)
        for p in range(4):
            a, b = 8 * g + 2 * p, 8 * g + 2 * p + 1
            if p in kept:
                row[a], row[b] = 2.0 + p, -(1.0 + p)
            else:
                row[a], row[b] = 0.25, 0.125
    row[0] = 8.0   # pair 0 of group 0: energy 64 + 1/64, above pair 1 (13) and pair 3 (41): pairs (0, 3) kept
    W = bf16(row[None, :])
    vals, meta, scales, st = orc.nvfp4_48_compress(W)
    nibs = [(meta[0, g // 2] >> (4 * (g % 2))) & 0xF for g in range(4)]
    assert nibs == [0 | (3 << 2), 0 | (2 << 2), 1 | (3 << 2), 0 | (2 << 2)]
    kept_vals = []
    for g, nib in enumerate(nibs):
        p0, p1 = nib & 3, nib >> 2
        kept_vals += [row[8 * g + 2 * p0], row[8 * g + 2 * p0 + 1], row[8 * g + 2 * p1], row[8 * g + 2 * p1 + 1]]
    amax = max(abs(v) for v in kept_vals)
    assert np.float32(st) == np.float32(amax) / np.float32(2688.0)
    codes = [(vals[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(16)]
    b = int(scales[0, 0])
    assert codes == [orc.nvfp4_code(float(v), b, st) for v in kept_vals]
    assert b == orc.nvfp4_block_code(float(amax), st)


# ---------------------------------------------------------------------------
# NVFP4 device images (layout spec): pinned by hand-derived positions and by
# being permutations of the canonical bytes plus fixed padding
# ---------------------------------------------------------------------------

def test_nvfp4_48_meta_image_positions_and_padding():
    rows, K = 200, 512
    g = np.random.default_rng(4)
    meta = g.integers(0, 256, size=(rows, K // 16), dtype=np.uint8)
    img = orc.nvfp4_48_meta_image(meta, rows, K)
    assert img.size == 2 * (K // 256) * 2048
    # row 5, positions 256..511 (chunk kc = 1): image row 5 of chunk (rb 0, kc 1)
    assert bytes(img[1 * 2048 + 16 * 5: 1 * 2048 + 16 * 6]) == bytes(meta[5, 16:32])
    # row 130 = block 1, image row 2, chunk (1, 0) at (1 * 2 + 0) * 2048
    assert bytes(img[2 * 2048 + 32: 2 * 2048 + 48]) == bytes(meta[130, 0:16])
    # rows past the end hold pairs 0 and 1 in every group
    assert (img[2 * 2048 + 16 * 72: 3 * 2048] == 0x44).all()
    # a permutation of the canonical bytes plus the padding
    live = np.concatenate([img[(rb * 2 + kc) * 2048 + 16 * L:(rb * 2 + kc) * 2048 + 16 * L + 16]
                           for rb in range(2) for L in range(128) if rb * 128 + L < rows for kc in range(2)])
    assert sorted(live.tolist()) == sorted(meta.ravel().tolist())


def test_nvfp4_scale_image_positions_and_padding():
    rows, nblk = 150, 8
    sc = np.random.default_rng(9).integers(1, 256, size=(rows, nblk), dtype=np.uint8)
    img = orc.nvfp4_scale_image(sc, rows)
    assert img.size == 256 * nblk
    # row 37 = 32 * 1 + 5 (q 1, l 5) of block 0, scale block 6 (kq 1, j 2)
    assert img[(0 * 2 + 1) * 512 + 16 * 5 + 4 * 1 + 2] == sc[37, 6]
    # row 140 = block 1, 32 * 0 + 12, scale block 3 (kq 0, j 3)
    assert img[(1 * 2 + 0) * 512 + 16 * 12 + 0 + 3] == sc[140, 3]
    # rows 150..255 hold 0; the live bytes are a permutation of the codes
    assert (img != 0).sum() == rows * nblk
    assert sorted(img[img != 0].tolist()) == sorted(sc.ravel().tolist())
