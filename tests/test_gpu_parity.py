"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: pruned/compressed values, the metadata image, E4M3 codes and
scales, decompression.  Within |y - y_ref| <= 2e-3 * sum_k |x_k w_k| + 1e-6:
GEMM outputs.  Shapes span several tiles plus ragged tails; the full-size
cases check sampled outputs."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from semi_structured_sparse_02_b200 import inputs, sp24
from tests.gpu_helpers import (OracleSparseW, bits16, check_tolerance, dev, dev_bf16, oracle_x,
                               u8, workspace_for)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# prune + compress (kernel 1), decompress, quantize
# ---------------------------------------------------------------------------

PRUNE_SHAPES = [(256, 256), (200, 384), (1, 128), (384, 1024), (130, 640)]


@pytest.mark.parametrize("rows,K", PRUNE_SHAPES)
def test_prune_compress_bf16_bit_exact(rows, K):
    W = inputs.weights_with_outliers(rows, K, seed=rows + K)
    ref = OracleSparseW(W, e4m3=False)
    Wd = dev_bf16(W)
    vals = torch.empty(rows, K // 2, dtype=torch.bfloat16, device="cuda")
    meta = torch.empty(sp24.meta_bytes(rows, K), dtype=torch.uint8, device="cuda")
    sp24.prune_compress(Wd, sp24.BF16, vals, meta)
    torch.cuda.synchronize()
    assert np.array_equal(bits16(vals), ref.values)
    assert np.array_equal(u8(meta), ref.image)
    dst = torch.empty(rows, K, dtype=torch.bfloat16, device="cuda")
    sp24.decompress(vals, meta, rows, K, sp24.BF16, dst)
    torch.cuda.synchronize()
    assert np.array_equal(bits16(dst), orc.decompress(ref.values, ref.canon, rows, K))


@pytest.mark.parametrize("rows,K", PRUNE_SHAPES)
def test_prune_compress_e4m3_bit_exact(rows, K):
    W = inputs.weights_with_outliers(rows, K, seed=7 * rows + K)
    ref = OracleSparseW(W, e4m3=True)
    Wd = dev_bf16(W)
    vals = torch.empty(rows, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(rows, K), dtype=torch.uint8, device="cuda")
    sc = torch.empty(rows, dtype=torch.float32, device="cuda")
    sp24.prune_compress(Wd, sp24.E4M3, vals, meta, row_scales=sc)
    torch.cuda.synchronize()
    assert np.array_equal(u8(vals), ref.values)
    assert np.array_equal(u8(meta), ref.image)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), ref.scales.view(np.uint32))
    dst = torch.empty(rows, K, dtype=torch.uint8, device="cuda")
    sp24.decompress(vals, meta, rows, K, sp24.E4M3, dst)
    torch.cuda.synchronize()
    assert np.array_equal(u8(dst), orc.decompress(ref.values, ref.canon, rows, K))


# the one-pass prune + cast kernel over each of its row mappings: 8, 7, 6, 5 or 4
# vectors per lane with no bounds checks (K = 4096, 1792, 1536 and 3072, 5120,
# 1024), 8 with checks (768, 25600), 256-thread CTAs of several rows and
# 512-thread CTAs of one (20480, 25600, 28672); ragged row counts; 30720 takes
# the amax / prune / scale passes
@pytest.mark.parametrize("rows,K", [(300, 4096), (130, 1792), (9, 1536), (37, 3072), (37, 5120), (200, 1024),
                                    (129, 768), (5, 20480), (3, 25600), (2, 28672), (3, 30720)])
def test_prune_compress_e4m3_one_pass_row_mappings(rows, K):
    W = inputs.weights_with_outliers(rows, K, seed=rows + 3 * K)
    W[0, :] = 0  # an all-zero row: scale 1, the metadata of zeros
    ref = OracleSparseW(W, e4m3=True)
    vals = torch.empty(rows, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(rows, K), dtype=torch.uint8, device="cuda")
    sc = torch.empty(rows, dtype=torch.float32, device="cuda")
    sp24.prune_compress(dev_bf16(W), sp24.E4M3, vals, meta, row_scales=sc)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    assert np.array_equal(u8(vals), ref.values)
    assert np.array_equal(u8(meta), ref.image)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), ref.scales.view(np.uint32))


def test_prune_handles_zero_rows_and_ties():
    W = np.zeros((128, 256), np.uint16)
    W[1, :8] = inputs.to_bf16_bits(np.array([1, 1, 1, 1, -2, 2, -2, 2], np.float32))
    W[2, :4] = inputs.to_bf16_bits(np.array([0, 0, 3, 0], np.float32))
    for e4 in (False, True):
        ref = OracleSparseW(W, e4m3=e4)
        vals = torch.empty(128, 128, dtype=torch.uint8 if e4 else torch.bfloat16, device="cuda")
        meta = torch.empty(sp24.meta_bytes(128, 256), dtype=torch.uint8, device="cuda")
        sc = torch.empty(128, dtype=torch.float32, device="cuda")
        sp24.prune_compress(dev_bf16(W), sp24.E4M3 if e4 else sp24.BF16, vals, meta,
                            row_scales=sc if e4 else None)
        torch.cuda.synchronize()
        assert np.array_equal(u8(meta), ref.image)
        got = u8(vals) if e4 else bits16(vals)
        assert np.array_equal(got, ref.values)
        if e4:
            assert np.array_equal(sc.cpu().numpy(), ref.scales)


@pytest.mark.parametrize("e4", [False, True])
def test_prune_hybrid_tiles_bit_exact(e4):
    rows, K = 384, 1024
    W = inputs.normal_bf16((rows, K), 0.02, seed=31)
    mask = inputs.hybrid_mask(rows, K, seed=31)
    ref = OracleSparseW(W, e4m3=e4, mask=mask)
    vals = torch.empty(rows, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device="cuda")
    meta = torch.empty(sp24.meta_bytes(rows, K), dtype=torch.uint8, device="cuda")
    dense = torch.zeros(rows, K, dtype=torch.uint8 if e4 else torch.bfloat16, device="cuda")
    sc = torch.empty(rows, dtype=torch.float32, device="cuda")
    sp24.prune_compress(dev_bf16(W), sp24.E4M3 if e4 else sp24.BF16, vals, meta,
                        row_scales=sc if e4 else None, tile_mask=dev(mask), dense_tiles=dense)
    torch.cuda.synchronize()
    assert np.array_equal(u8(meta), ref.image)
    if e4:
        assert np.array_equal(u8(vals), ref.values)
        assert np.array_equal(u8(dense), ref.dense)
        assert np.array_equal(sc.cpu().numpy(), ref.scales)
    else:
        assert np.array_equal(bits16(vals), ref.values)
        assert np.array_equal(bits16(dense), ref.dense)


# register-resident warp segments up to 28672 wide (one warp per 1792 elements:
# 37 x 1792 packs 16 rows per CTA with a ragged last CTA, 28672 fills 16 warps);
# the two-pass kernel beyond (30720)
@pytest.mark.parametrize("rows,K", [(1, 5120), (16, 256), (128, 4096), (7, 25600), (37, 1792), (2, 28672),
                                    (3, 30720)])
def test_quantize_rows_e4m3_bit_exact(rows, K):
    X = inputs.normal_bf16((rows, K), 1.0, seed=rows * 3 + K)
    X[0, :] = 0  # an all-zero token: scale 1, codes 0
    q_ref, s_ref = orc.quantize_rows_e4m3(X)
    q = torch.empty(rows, K, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    sp24.quantize_e4m3_rows(dev_bf16(X), q, s)
    torch.cuda.synchronize()
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("shapes", [
    [(1, 5120), (8, 25600), (32, 256), (128, 4096), (5, 28672)],   # warp-segment kernel
    [(1, 5120), (8, 25600), (32, 256), (128, 4096), (3, 33024)],   # a row too long for it: two-pass kernel
])
def test_grouped_quantize_matches_oracle_per_matrix(shapes):
    pairs, refs = [], []
    for i, (rows, K) in enumerate(shapes):
        X = inputs.normal_bf16((rows, K), 1.0, seed=50 + i)
        refs.append(orc.quantize_rows_e4m3(X))
        pairs.append((dev_bf16(X), torch.empty(rows, K, dtype=torch.uint8, device="cuda"),
                      torch.empty(rows, dtype=torch.float32, device="cuda")))
    g = sp24.QuantGroup(pairs)
    g()
    torch.cuda.synchronize()
    for (src, q, s), (q_ref, s_ref) in zip(pairs, refs):
        assert np.array_equal(u8(q), q_ref)
        assert np.array_equal(s.cpu().numpy(), s_ref)


# ---------------------------------------------------------------------------
# GEMM (kernels 2 and 3)
# ---------------------------------------------------------------------------

GEMM_SHAPES = [
    (16, 256, 256),     # the tiny configuration
    (1, 384, 512),
    (40, 256, 1280),
    (130, 512, 768),    # two token tiles, ragged
    (8, 1024, 4096),    # decode-like: split-K
    (256, 384, 384),
]


def prepare_gemm(X_bits, W_bits, e4, tactic, out_f32, mask=None, flags=0):
    """Device operands from the oracle's own compression and quantization, the
    argument block, and the oracle's fp64 product with its error scale."""
    M, K = X_bits.shape
    N = W_bits.shape[0]
    xq, xs, X_hat = oracle_x(X_bits, e4)
    Xd = dev(xq) if e4 else dev_bf16(xq)
    Y = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    if tactic == sp24.SPARSE:
        ref = OracleSparseW(W_bits, e4m3=e4, mask=mask)
        Wd = dev(ref.values) if e4 else dev_bf16(ref.values)
        W_hat = ref.W_hat
        a = sp24.gemm_args(Xd, Wd, Y, K, sp24.SPARSE, W_meta=dev(ref.image),
                           x_scales=dev(xs) if e4 else None,
                           w_scales=dev(ref.scales) if e4 else None,
                           tile_mask=dev(mask) if mask is not None else None,
                           W_dense_tiles=dev(ref.dense) if mask is not None else None)
    else:
        if e4:
            wq, ws_ = orc.quantize_rows_e4m3(W_bits)
            Wd = dev(wq)
            W_hat = orc.e4m3_decode(wq) * ws_.astype(np.float64)[:, None]
        else:
            ws_ = None
            Wd = dev_bf16(W_bits)
            W_hat = orc.bf16_bits_to_f64(W_bits)
        a = sp24.gemm_args(Xd, Wd, Y, K, sp24.DENSE, x_scales=dev(xs) if e4 else None,
                           w_scales=dev(ws_) if e4 else None)
    a.flags = flags
    y_ref, a_ref = orc.gemm_f64(X_hat, W_hat)
    return a, Y, y_ref, a_ref


def run_gemm(X_bits, W_bits, e4, tactic, out_f32, mask=None, use_ws=True, flags=0):
    a, Y, y_ref, a_ref = prepare_gemm(X_bits, W_bits, e4, tactic, out_f32, mask, flags)
    ws = workspace_for(a) if use_ws else None
    sp24.set_workspace(a, ws)
    sp24.gemm(a)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    return Y.float().cpu().numpy().astype(np.float64), y_ref, a_ref, a, ws


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("e4", [False, True])
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_gemm_parity(M, N, K, e4, tactic):
    X, W = inputs.linear_pair(M, N, K, seed=M + N + K, outliers=True)
    for out_f32 in (True, False):
        y, y_ref, a_ref, _, _ = run_gemm(X, W, e4, tactic, out_f32)
        check_tolerance(y, y_ref, a_ref, "M%d N%d K%d e4=%s tactic=%d f32=%s" % (M, N, K, e4, tactic, out_f32))


@pytest.mark.parametrize("M,N,K", [(16, 200, 256), (3, 72, 128), (33, 136, 96)])
def test_dense_gemm_ragged_n(M, N, K):
    X, W = inputs.linear_pair(M, N, K, seed=5)
    for e4 in (False, True):
        y, y_ref, a_ref, _, _ = run_gemm(X, W, e4, sp24.DENSE, True)
        check_tolerance(y, y_ref, a_ref, "dense ragged")


@pytest.mark.parametrize("M,N,K", [(8, 1024, 4096), (1, 384, 512), (40, 256, 1280), (128, 640, 2048)])
@pytest.mark.parametrize("e4", [False, True])
def test_whole_tile_schedule_without_workspace(M, N, K, e4):
    X, W = inputs.linear_pair(M, N, K, seed=3 * M + N)
    y, y_ref, a_ref, _, ws = run_gemm(X, W, e4, sp24.SPARSE, True, use_ws=False)
    assert ws is None
    check_tolerance(y, y_ref, a_ref, "whole tiles")


@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_stream_k_workspace_is_reusable(tactic):
    # three calls on one workspace: every call leaves the accumulators and
    # counters zero, so each one is within tolerance on its own (a residue
    # would add a whole partial sum); the split tiles' fp32 addition order may
    # differ between calls, so they agree to fp32 rounding
    X, W = inputs.linear_pair(8, 1024, 4096, seed=77)
    y1, y_ref, a_ref, args, ws = run_gemm(X, W, True, tactic, True, flags=sp24.GEMM_W_STATIC)
    assert ws is not None  # this decode shape takes the stream-K schedule
    check_tolerance(y1, y_ref, a_ref, "stream-K")
    Y = args._keep[2]
    for _ in range(2):
        Y.zero_()
        sp24.gemm(args)
        torch.cuda.synchronize()
        y = Y.cpu().numpy().astype(np.float64)
        check_tolerance(y, y_ref, a_ref, "stream-K repeat")
        assert np.allclose(y, y1, rtol=1e-5, atol=1e-5 * np.abs(y1).max())
    nstate = sp24.gemm_workspace_state_bytes(args)
    assert 0 < nstate <= ws.numel()
    assert int(ws[:nstate].view(torch.int32).abs().sum().item()) == 0  # counters and flags zero


@pytest.mark.parametrize("M,N,K", [(1, 5120, 5120), (32, 2560, 25600), (128, 1280, 5120)])
def test_w_static_prefetch_parity(M, N, K):
    X, W = inputs.linear_pair(M, N, K, seed=M + 11)
    y, y_ref, a_ref, _, _ = run_gemm(X, W, True, sp24.SPARSE, False, flags=sp24.GEMM_W_STATIC)
    check_tolerance(y, y_ref, a_ref, "w_static")


# Grouped launches: independent problems of one M class, different N and K,
# with ragged token counts; each output is checked against the oracle.
GROUPS = {
    "decode": [(8, 1024, 4096), (5, 384, 512), (16, 640, 2048), (1, 256, 1280)],
    "m32": [(17, 512, 1024), (32, 256, 3072), (20, 1152, 256)],
    "m64": [(40, 256, 1280), (64, 768, 512)],
    "m128": [(130, 512, 768), (256, 384, 384), (65, 128, 2560)],
}


def run_group(shapes, e4, tactic, out_f32, use_ws=True, flags=0, seed=0):
    items = []
    for i, (M, N, K) in enumerate(shapes):
        X, W = inputs.linear_pair(M, N, K, seed=seed + 31 * i + M, outliers=True)
        items.append(prepare_gemm(X, W, e4, tactic, out_f32, flags=flags))
    grp = sp24.GemmGroup([it[0] for it in items], allocate_workspace=use_ws)
    grp()
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    return grp, items


def check_group(items, what):
    for i, (_, Y, y_ref, a_ref) in enumerate(items):
        y = Y.float().cpu().numpy().astype(np.float64)
        check_tolerance(y, y_ref, a_ref, "%s problem %d" % (what, i))


@pytest.mark.parametrize("group", sorted(GROUPS))
@pytest.mark.parametrize("e4", [False, True])
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_grouped_gemm_parity(group, e4, tactic):
    for out_f32 in (True, False):
        _, items = run_group(GROUPS[group], e4, tactic, out_f32, seed=len(group))
        check_group(items, "group %s e4=%s tactic=%d f32=%s" % (group, e4, tactic, out_f32))


# Groups whose problems come from different token-count classes: the launch
# takes the widest class's tile, each problem runs its own width.
MIXED_GROUPS = {
    "to32": [(1, 512, 1024), (8, 384, 2048), (32, 640, 1024), (20, 256, 512)],
    "to128": [(1, 256, 1024), (16, 384, 512), (32, 512, 1536), (128, 640, 1024), (100, 256, 2048)],
}


@pytest.mark.parametrize("group", sorted(MIXED_GROUPS))
@pytest.mark.parametrize("e4", [False, True])
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
@pytest.mark.parametrize("use_ws", [True, False])
def test_grouped_gemm_mixed_token_classes(group, e4, tactic, use_ws):
    for out_f32 in (True, False):
        _, items = run_group(MIXED_GROUPS[group], e4, tactic, out_f32, use_ws=use_ws, seed=len(group) + 5,
                             flags=sp24.GEMM_W_STATIC)
        check_group(items, "mixed group %s e4=%s tactic=%d ws=%s f32=%s" % (group, e4, tactic, use_ws, out_f32))


@pytest.mark.parametrize("group", ["decode", "to32"])
def test_stream_k_split_is_fixed_and_repeats_bitwise(group):
    """A split tile is finished by the unit that holds its first K-stage, so the
    split and the fp32 addition order depend only on the plan: repeated calls
    (and a call after other launches on the same workspace) give identical
    bytes, and agree with the oracle."""
    shapes = GROUPS[group] if group in GROUPS else MIXED_GROUPS[group]
    grp, items = run_group(shapes, True, sp24.SPARSE, True, seed=11)
    assert grp.workspace_bytes() > 0  # the stream-K schedule, with split tiles
    first = [Y.clone() for (_, Y, _, _) in items]
    for _ in range(3):
        for (_, Y, _, _) in items:
            Y.fill_(float("nan"))
        grp()
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        for y0, (_, Y, _, _) in zip(first, items):
            assert torch.equal(y0.view(torch.int32), Y.view(torch.int32))
    check_group(items, "stream-K repeat %s" % group)


@pytest.mark.parametrize("e4", [False, True])
def test_grouped_gemm_whole_tiles_without_workspace(e4):
    grp, items = run_group(GROUPS["decode"], e4, sp24.SPARSE, True, use_ws=False)
    assert grp.workspace_bytes() > 0  # stream-K would have been chosen with a workspace
    check_group(items, "grouped whole tiles")


def test_independent_group_chain_after_one_cast():
    """A per-token cast, then three grouped launches of independent GEMMs on one
    stream, the second and third flagged as following an independent GEMM
    launch (they start before the previous group finishes and wait for it only
    before exiting).  Every iteration casts different activations and writes
    its own outputs, with no host synchronization in between, so a group that
    read its activations before the cast finished would show the previous
    iteration's values."""
    classes = [[(1, 512, 1024), (8, 384, 2048)], [(32, 640, 1024)], [(128, 512, 1536), (100, 256, 1024)]]
    iters = 4
    torch.cuda.synchronize()
    shapes = [sh for cl in classes for sh in cl]
    Ws = [OracleSparseW(inputs.normal_bf16((N, K), 0.02, seed=100 + j), e4m3=True) for j, (_, N, K) in enumerate(shapes)]
    Wd = [(dev(w.values), dev(w.image), dev(w.scales)) for w in Ws]
    srcs = [[inputs.normal_bf16((M, K), 1.0, seed=1000 * t + j) for j, (M, _, K) in enumerate(shapes)]
            for t in range(iters)]
    xb = [[dev_bf16(x) for x in it] for it in srcs]
    xq = [torch.empty(M, K, dtype=torch.uint8, device="cuda") for (M, _, K) in shapes]
    xs = [torch.empty(M, dtype=torch.float32, device="cuda") for (M, _, _) in shapes]
    Ys = [[torch.empty(M, N, dtype=torch.float32, device="cuda") for (M, N, _) in shapes] for _ in range(iters)]
    # groups (and their workspaces) built first, so that the launches below
    # follow one another directly in the stream
    casts, groups = [], []
    for t in range(iters):
        casts.append(sp24.QuantGroup([(xb[t][j], xq[j], xs[j]) for j in range(len(shapes))]))
        j0, gt = 0, []
        for c, cl in enumerate(classes):
            args = []
            for j in range(j0, j0 + len(cl)):
                v, m, sc = Wd[j]
                args.append(sp24.gemm_args(xq[j], v, Ys[t][j], shapes[j][2], sp24.SPARSE, W_meta=m,
                                           x_scales=xs[j], w_scales=sc, flags=sp24.GEMM_W_STATIC))
            gt.append(sp24.GemmGroup(args, after_independent=c > 0))
            j0 += len(cl)
        groups.append(gt)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for t in range(iters):
            casts[t](stream)
            for grp in groups[t]:
                grp(stream)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    for t in range(iters):
        for j, (M, N, K) in enumerate(shapes):
            _, _, X_hat = oracle_x(srcs[t][j], True)
            y_ref, a_ref = orc.gemm_f64(X_hat, Ws[j].W_hat)
            check_tolerance(Ys[t][j].cpu().numpy().astype(np.float64), y_ref, a_ref,
                            "iteration %d problem %d" % (t, j))


def test_grouped_gemm_sixteen_problems_w_static_reusable():
    # the largest group: 16 decode projections of mixed sizes, weights marked
    # static; three calls on one workspace, which ends zero after each
    shapes = [(1 + (i % 16), 128 * (1 + i % 5), 256 * (1 + (i * 7) % 9)) for i in range(16)]
    grp, items = run_group(shapes, True, sp24.SPARSE, True, flags=sp24.GEMM_W_STATIC, seed=5)
    check_group(items, "16 problems")
    first = [it[1].clone() for it in items]
    for _ in range(2):
        for it in items:
            it[1].zero_()
        grp()
        torch.cuda.synchronize()
        check_group(items, "16 problems repeat")
        for it, y1 in zip(items, first):
            y1 = y1.cpu().numpy().astype(np.float64)
            assert np.allclose(it[1].cpu().numpy(), y1, rtol=1e-5, atol=1e-5 * np.abs(y1).max())
    if grp.workspace is not None:
        nstate = grp.workspace_state_bytes()
        assert int(grp.workspace[:nstate].view(torch.int32).abs().sum().item()) == 0


@pytest.mark.parametrize("e4", [False, True])
def test_grouped_gemm_cta_pairs(e4):
    # the decode group on CTA pairs (ragged N: 384 and 640 leave the second
    # CTA of the last pair tile past the end)
    shapes = [(8, 1024, 4096), (5, 384, 512), (16, 640, 2048), (1, 256, 1280)]
    flags = sp24.GEMM_CTA_PAIR | sp24.GEMM_W_STATIC
    for use_ws in (True, False):
        _, items = run_group(shapes, e4, sp24.SPARSE, True, use_ws=use_ws, flags=flags, seed=17)
        check_group(items, "pair group ws=%s" % use_ws)


def test_launch_cache_tells_argument_sets_apart():
    # repeated calls with identical arguments reuse a cached launch; any
    # changed field (here the output pointer, then the workspace) must not
    X, W = inputs.linear_pair(8, 1024, 4096, seed=321)
    a, Y1, y_ref, a_ref = prepare_gemm(X, W, True, sp24.SPARSE, True)
    for _ in range(2):
        Y1.zero_()
        sp24.gemm(a)
        torch.cuda.synchronize()
        check_tolerance(Y1.cpu().numpy().astype(np.float64), y_ref, a_ref, "cached call")
    Y2 = torch.zeros_like(Y1)
    b = sp24.gemm_args(a._keep[0], a._keep[1], Y2, 4096, sp24.SPARSE, W_meta=a._keep[3], x_scales=a._keep[4],
                       w_scales=a._keep[5])
    Y1.zero_()
    sp24.gemm(b)
    torch.cuda.synchronize()
    assert float(Y1.abs().max()) == 0.0
    check_tolerance(Y2.cpu().numpy().astype(np.float64), y_ref, a_ref, "new output pointer")
    ws = workspace_for(b)
    assert ws is not None
    sp24.set_workspace(b, ws)  # stream-K schedule now: a different launch
    Y2.zero_()
    sp24.gemm(b)
    torch.cuda.synchronize()
    check_tolerance(Y2.cpu().numpy().astype(np.float64), y_ref, a_ref, "with workspace")
    nstate = sp24.gemm_workspace_state_bytes(b)
    assert int(ws[:nstate].view(torch.int32).abs().sum().item()) == 0


def test_group_of_one_matches_single_gemm():
    X, W = inputs.linear_pair(8, 1024, 4096, seed=123)
    a, Y, y_ref, a_ref = prepare_gemm(X, W, True, sp24.SPARSE, True)
    sp24.gemm_grouped([a])
    torch.cuda.synchronize()
    yg = Y.cpu().numpy().astype(np.float64)
    check_tolerance(yg, y_ref, a_ref, "group of one")
    sp24.set_workspace(a, workspace_for(a))
    Y.zero_()
    sp24.gemm(a)
    torch.cuda.synchronize()
    assert np.allclose(Y.cpu().numpy(), yg, rtol=1e-5, atol=1e-5 * np.abs(yg).max())


@pytest.mark.parametrize("M", [1, 16, 200])
def test_hybrid_gemm_parity(M):
    N, K = 512, 1024
    X, W = inputs.linear_pair(M, N, K, seed=M + 3)
    mask = inputs.hybrid_mask(N, K, seed=M)
    y, y_ref, a_ref, _, _ = run_gemm(X, W, True, sp24.SPARSE, True, mask=mask)
    check_tolerance(y, y_ref, a_ref, "hybrid")


# Grouped launches of hybrid weights (one-CTA tiles): a token-count class of
# qkv / o / gate_up / down-like shapes.  K = 5120 gives 40 K-steps per tile, so
# a segment spans more than one 32-step word of dense flags.
HYBRID_GROUPS = {
    "decode": [(1, 768, 512), (16, 512, 1024), (5, 1536, 512), (9, 256, 5120)],
    "m128": [(256, 768, 512), (200, 512, 1536), (70, 384, 5120)],
}


def _group_mask(kind, N, K, seed):
    RB, KT = N // 128, K // 128
    if kind == "random":
        return inputs.hybrid_mask(N, K, seed=seed)
    if kind == "all_dense":
        return np.ones((RB, KT), np.uint8)
    return ((np.arange(RB)[:, None] + np.arange(KT)[None, :]) % 2).astype(np.uint8)


@pytest.mark.parametrize("group", sorted(HYBRID_GROUPS))
@pytest.mark.parametrize("use_ws", [True, False])
@pytest.mark.parametrize("kind", ["random", "all_dense", "checkerboard"])
def test_grouped_hybrid_gemm_parity(group, use_ws, kind):
    shapes = HYBRID_GROUPS[group]
    items = []
    for i, (M, N, K) in enumerate(shapes):
        X, W = inputs.linear_pair(M, N, K, seed=17 * i + M + K, outliers=True)
        mask = _group_mask(kind, N, K, seed=i + M)
        items.append(prepare_gemm(X, W, True, sp24.SPARSE, True, mask=mask, flags=sp24.GEMM_W_STATIC))
    grp = sp24.GemmGroup([it[0] for it in items], allocate_workspace=use_ws)
    if use_ws and group == "decode":
        assert grp.ws_bytes > 0  # the stream-K schedule
    for call in range(2):  # the second call reuses the workspace the first left zeroed
        for it in items:
            it[1].fill_(float("nan"))
        grp()
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        check_group(items, "hybrid group %s ws=%s %s call %d" % (group, use_ws, kind, call))


def test_grouped_hybrid_first_call_inside_stream_capture():
    """A hybrid group whose first call is made while its stream is being
    captured into a CUDA graph: the planner skips reading the tile masks back
    (the schedule is then cut by stage counts alone) and the replayed graph
    still gives the oracle's results; later eager calls reuse that plan."""
    shapes = [(1, 768, 1024), (16, 512, 2048), (8, 1536, 512)]
    items = []
    for i, (M, N, K) in enumerate(shapes):
        X, W = inputs.linear_pair(M, N, K, seed=41 * i + M + K, outliers=True)
        items.append(prepare_gemm(X, W, True, sp24.SPARSE, True, mask=inputs.hybrid_mask(N, K, seed=3 + i),
                                  flags=sp24.GEMM_W_STATIC))
    grp = sp24.GemmGroup([it[0] for it in items])  # workspace allocated before the capture
    assert grp.ws_bytes > 0  # the stream-K schedule, whose cut reads the masks when it can
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        grp(stream=stream)
    for _ in range(2):
        for it in items:
            it[1].fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        check_group(items, "hybrid group, first call captured")
    for it in items:
        it[1].fill_(float("nan"))
    grp()
    torch.cuda.synchronize()
    check_group(items, "hybrid group, eager call after the capture")


def test_grouped_hybrid_mixed_token_classes():
    shapes = [(1, 768, 512), (16, 512, 1024), (32, 256, 5120), (100, 384, 640)]
    items = []
    for i, (M, N, K) in enumerate(shapes):
        X, W = inputs.linear_pair(M, N, K, seed=29 * i + M + K, outliers=True)
        items.append(prepare_gemm(X, W, True, sp24.SPARSE, False, mask=inputs.hybrid_mask(N, K, seed=i),
                                  flags=sp24.GEMM_W_STATIC))
    for use_ws in (True, False):
        grp = sp24.GemmGroup([it[0] for it in items], allocate_workspace=use_ws)
        grp()
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        check_group(items, "hybrid mixed classes ws=%s" % use_ws)


def test_grouped_rejects_mixed_hybrid_and_plain_weights():
    X, W = inputs.linear_pair(8, 256, 512, seed=3)
    plain = prepare_gemm(X, W, True, sp24.SPARSE, True)[0]
    hyb = prepare_gemm(X, W, True, sp24.SPARSE, True, mask=inputs.hybrid_mask(256, 512, seed=1))[0]
    arr = (sp24.GemmArgs * 2)(plain, hyb)
    st = sp24.lib().sp24_gemm_grouped(arr, 2, None, 0, None)
    assert st == sp24.SP24_ERR_INVALID_ARG


@pytest.mark.parametrize("M,N,K", [(8, 256, 640), (130, 384, 128), (1, 128, 1152), (33, 512, 1536)])
@pytest.mark.parametrize("kind", ["random", "checkerboard", "all_dense", "all_sparse", "odd_columns"])
def test_hybrid_stage_kinds(M, N, K, kind):
    """One-CTA hybrid stages cover two tile columns: both sparse, both dense,
    mixed either way, and a single last column when K / 128 is odd."""
    RB, KT = N // 128, K // 128
    if kind == "random":
        mask = inputs.hybrid_mask(N, K, seed=K)
    elif kind == "checkerboard":
        mask = ((np.arange(RB)[:, None] + np.arange(KT)[None, :]) % 2).astype(np.uint8)
    elif kind == "all_dense":
        mask = np.ones((RB, KT), np.uint8)
    elif kind == "all_sparse":
        mask = np.zeros((RB, KT), np.uint8)
    else:  # every odd column dense: each stage is sparse then dense
        mask = np.zeros((RB, KT), np.uint8)
        mask[:, 1::2] = 1
    X, W = inputs.linear_pair(M, N, K, seed=M + N + K, outliers=True)
    for use_ws in (True, False):
        y, y_ref, a_ref, _, _ = run_gemm(X, W, True, sp24.SPARSE, True, mask=mask, use_ws=use_ws,
                                         flags=sp24.GEMM_W_STATIC | sp24.GEMM_SINGLE_CTA)
        check_tolerance(y, y_ref, a_ref, "hybrid kinds %s M%d N%d K%d ws=%s" % (kind, M, N, K, use_ws))


def _pair_mask(kind, N, K, seed):
    RB, KT = N // 128, K // 128
    if kind == "random":
        return inputs.hybrid_mask(N, K, seed=seed)
    if kind == "all_dense":
        return np.ones((RB, KT), np.uint8)
    if kind == "all_sparse":
        return np.zeros((RB, KT), np.uint8)
    if kind == "odd_blocks":   # every pair mixed: the second half dense, the first sparse
        m = np.zeros((RB, KT), np.uint8)
        m[1::2, :] = 1
        return m
    if kind == "checkerboard":  # mixed, dense-first and dense-second K-steps interleaved
        return ((np.arange(RB)[:, None] + np.arange(KT)[None, :]) % 2).astype(np.uint8)
    raise ValueError(kind)


HYBRID_PAIR_SHAPES = [
    (256, 512, 1024),
    (300, 384, 640),    # ragged token tile; the last weight tile's second half is past the end
    (520, 768, 2048),
]


@pytest.mark.parametrize("M,N,K", HYBRID_PAIR_SHAPES)
@pytest.mark.parametrize("kind", ["random", "all_dense", "all_sparse", "odd_blocks", "checkerboard"])
def test_hybrid_gemm_pair_parity(M, N, K, kind):
    """Hybrid weights on CTA pairs (forced: these shapes have fewer tiles than
    the device has pairs), where a K-step runs dense when either half of the
    pair is dense there.  Checked against the oracle and against the one-CTA
    kernel."""
    X, W = inputs.linear_pair(M, N, K, seed=M + N + K + 7, outliers=True)
    mask = _pair_mask(kind, N, K, seed=M + K)
    y, y_ref, a_ref, _, _ = run_gemm(X, W, True, sp24.SPARSE, True, mask=mask, flags=sp24.GEMM_CTA_PAIR)
    check_tolerance(y, y_ref, a_ref, "hybrid pair %s M%d N%d K%d" % (kind, M, N, K))
    y1, _, _, _, _ = run_gemm(X, W, True, sp24.SPARSE, True, mask=mask, flags=sp24.GEMM_SINGLE_CTA)
    scale = np.abs(y_ref).max()
    assert np.allclose(y, y1, rtol=1e-5, atol=1e-5 * scale)


def test_hybrid_pair_gemm_on_gpu_pruned_weights():
    """The device prune writes the dense-form array the pair kernel reads at
    mixed K-steps; the whole chain against the oracle."""
    M, N, K = 512, 640, 1536
    X, W = inputs.linear_pair(M, N, K, seed=17, outliers=True)
    mask = inputs.hybrid_mask(N, K, seed=17)
    ref = OracleSparseW(W, e4m3=True, mask=mask)
    vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    dense = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    sc = torch.empty(N, dtype=torch.float32, device="cuda")
    sp24.prune_compress(dev_bf16(W), sp24.E4M3, vals, meta, row_scales=sc, tile_mask=dev(mask), dense_tiles=dense)
    torch.cuda.synchronize()
    assert np.array_equal(u8(dense), ref.dense)
    xq, xs, X_hat = oracle_x(X, True)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    a = sp24.gemm_args(dev(xq), vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=dev(xs), w_scales=sc,
                       tile_mask=dev(mask), W_dense_tiles=dense)
    a.flags = sp24.GEMM_CTA_PAIR
    sp24.gemm(a)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    y_ref, a_ref = orc.gemm_f64(X_hat, ref.W_hat)
    check_tolerance(Y.cpu().numpy().astype(np.float64), y_ref, a_ref, "hybrid pair, device-pruned W")


def test_gemm_with_gpu_pruned_weights_end_to_end():
    M, N, K = 32, 640, 2048
    X, W = inputs.linear_pair(M, N, K, seed=9, outliers=True)
    Wd = dev_bf16(W)
    vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    ws_ = torch.empty(N, dtype=torch.float32, device="cuda")
    sp24.prune_compress(Wd, sp24.E4M3, vals, meta, row_scales=ws_)
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sp24.quantize_e4m3_rows(dev_bf16(X), xq, xs)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.gemm_args(xq, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=ws_)
    ws = workspace_for(a)
    sp24.set_workspace(a, ws)
    sp24.gemm(a)
    torch.cuda.synchronize()
    ref = OracleSparseW(W, e4m3=True)
    _, _, X_hat = oracle_x(X, True)
    y_ref, a_ref = orc.gemm_f64(X_hat, ref.W_hat)
    check_tolerance(Y.float().cpu().numpy().astype(np.float64), y_ref, a_ref, "end to end")


# ---------------------------------------------------------------------------
# online activation prune + compress fused ahead of the GEMM (kernel 4)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(128, 384, 512), (200, 256, 1024), (1, 128, 128)])
def test_activation_fused_parity(M, N, K):
    X = inputs.student_t_bf16((M, K), 3.0, seed=M + K)
    W = inputs.normal_bf16((N, K), 0.02, seed=N)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    xv = torch.empty(M, K // 2, dtype=torch.bfloat16, device="cuda")
    xm = torch.empty(sp24.meta_bytes(M, K), dtype=torch.uint8, device="cuda")
    sp24.prune_compress_activations_fused(dev_bf16(X), dev_bf16(W), Y, x_values=xv, x_meta=xm)
    torch.cuda.synchronize()
    pruned, vals, canon = orc.prune_compress_bf16(X)
    assert np.array_equal(bits16(xv), vals)
    assert np.array_equal(u8(xm), orc.meta_image(canon, M, K, False))
    y_ref, a_ref = orc.gemm_f64(orc.bf16_bits_to_f64(pruned), orc.bf16_bits_to_f64(W))
    check_tolerance(Y.cpu().numpy().astype(np.float64), y_ref, a_ref, "activations")
    # workspace variant, bf16 output
    ws = torch.empty(sp24.activations_workspace_bytes(M, K), dtype=torch.uint8, device="cuda")
    Y2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sp24.prune_compress_activations_fused(dev_bf16(X), dev_bf16(W), Y2, workspace=ws)
    torch.cuda.synchronize()
    check_tolerance(Y2.float().cpu().numpy().astype(np.float64), y_ref, a_ref, "activations ws")


# ---------------------------------------------------------------------------
# CTA-pair kernel (M >= 256 and N >= 256): 256 x 256 tiles on two SMs
# ---------------------------------------------------------------------------
PAIR_SHAPES = [
    (256, 256, 256),     # one pair tile
    (512, 384, 1024),    # second row tile half past N: zero-filled A rows, clamped metadata
    (300, 640, 768),     # ragged token count
    (260, 256, 384),     # e4m3: the last 256-deep stage holds one 128-deep chunk
    (1024, 1024, 2048),  # 16 tiles, deep K
]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
@pytest.mark.parametrize("e4", [False, True])
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_pair_kernel_parity(M, N, K, e4, tactic):
    X, W = inputs.linear_pair(M, N, K, seed=7 * M + N + K, outliers=True)
    for out_f32 in (True, False):
        y, y_ref, a_ref, args, ws = run_gemm(X, W, e4, tactic, out_f32)
        assert ws is None  # the pair kernel needs no workspace
        check_tolerance(y, y_ref, a_ref, "pair M%d N%d K%d e4=%s tactic=%d f32=%s"
                        % (M, N, K, e4, tactic, out_f32))
    # the one-CTA kernel on the same operands agrees to the same tolerance
    y1, _, _, _, _ = run_gemm(X, W, e4, tactic, True, flags=sp24.GEMM_SINGLE_CTA)
    check_tolerance(y1, y_ref, a_ref, "single-CTA M%d N%d K%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", [(1, 384, 2048), (8, 1024, 4096), (16, 2560, 1280), (40, 640, 768),
                                   (128, 1280, 5120)])
@pytest.mark.parametrize("e4", [False, True])
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_decode_pair_tiles_and_single_cta_agree(M, N, K, e4, tactic):
    # with GEMM_CTA_PAIR, M <= 255 and N >= 256 run 256-row tiles on CTA pairs
    # (stream-K when the tiles are few); the default one-CTA tiles must agree
    # to the same tolerance
    X, W = inputs.linear_pair(M, N, K, seed=M * 3 + N, outliers=True)
    pair = sp24.GEMM_CTA_PAIR
    for flags in (0, sp24.GEMM_W_STATIC, pair, pair | sp24.GEMM_W_STATIC):
        y, y_ref, a_ref, _, _ = run_gemm(X, W, e4, tactic, True, flags=flags)
        check_tolerance(y, y_ref, a_ref, "decode M%d N%d K%d e4=%s tactic=%d flags=%d"
                        % (M, N, K, e4, tactic, flags))


@pytest.mark.parametrize("e4", [False, True])
def test_pair_kernel_many_tiles_per_pair_sampled(e4):
    # 4096 x 4096 output = 256 tiles over at most 74 pairs: every pair runs
    # several tiles, cycling both accumulators (and, sparse, their overlap)
    M, N, K = 4096, 4096, 512
    X, W = inputs.linear_pair(M, N, K, seed=99, outliers=True)
    for tactic in (sp24.SPARSE, sp24.DENSE):
        a, Y, _, _ = _prepare_large(X, W, e4, tactic)
        sp24.gemm(a)
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        g = np.random.default_rng(3)
        ms = np.concatenate([g.choice(M, size=40, replace=False), [0, 255, 256, M - 1]])
        ns = np.concatenate([g.choice(N, size=40, replace=False), [0, 255, 256, N - 1]])
        W_hat = _w_hat(W[ns], e4, tactic)
        _, _, X_hat = oracle_x(X[ms], e4)
        y_ref, a_ref = orc.gemm_f64_sampled(X_hat, W_hat, np.arange(ms.size), np.arange(ns.size))
        y_gpu = Y.float().cpu().numpy().astype(np.float64)[np.ix_(ms, ns)].diagonal()
        check_tolerance(y_gpu, y_ref, a_ref, "pair many tiles e4=%s tactic=%d" % (e4, tactic))


def _w_hat(W_rows, e4, tactic):
    if tactic == sp24.SPARSE:
        return OracleSparseW(W_rows, e4m3=e4).W_hat
    if e4:
        wq, s = orc.quantize_rows_e4m3(W_rows)
        return orc.e4m3_decode(wq) * s.astype(np.float64)[:, None]
    return orc.bf16_bits_to_f64(W_rows)


def _prepare_large(X_bits, W_bits, e4, tactic):
    """Device operands from the library's own prune / quantize (bit-exact to
    the oracle, checked elsewhere), for sizes where the oracle's full
    compression would be slow."""
    M, K = X_bits.shape
    N = W_bits.shape[0]
    Wd = dev_bf16(W_bits)
    ws_ = torch.empty(N, dtype=torch.float32, device="cuda") if e4 else None
    if tactic == sp24.SPARSE:
        Wv = torch.empty(N, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device="cuda")
        meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
        sp24.prune_compress(Wd, sp24.E4M3 if e4 else sp24.BF16, Wv, meta, row_scales=ws_)
    else:
        meta = None
        if e4:
            Wv = torch.empty(N, K, dtype=torch.uint8, device="cuda")
            sp24.quantize_e4m3_rows(Wd, Wv, ws_)
        else:
            Wv = Wd
    if e4:
        Xd = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        xs = torch.empty(M, dtype=torch.float32, device="cuda")
        sp24.quantize_e4m3_rows(dev_bf16(X_bits), Xd, xs)
    else:
        Xd, xs = dev_bf16(X_bits), None
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.gemm_args(Xd, Wv, Y, K, tactic, W_meta=meta, x_scales=xs, w_scales=ws_)
    return a, Y, None, None


@pytest.mark.parametrize("M,N,K", [(128, 384, 512), (200, 256, 1280), (1, 128, 128), (512, 384, 512),
                                   (300, 640, 768), (37, 128, 4096), (20, 128, 5120), (3, 128, 20480),
                                   (2, 128, 25600), (5, 256, 32768)])
def test_activation_fused_e4m3_parity(M, N, K):
    # rows up to 28672 wide take the one-pass kernel (row in registers); the
    # 32768-wide case takes the amax / prune / scale passes
    # X pruned 2:4 and cast to e4m3 per token on every call; the compressed
    # activations are bit-exact to the oracle's, Y within tolerance
    X = inputs.student_t_bf16((M, K), 3.0, seed=M + 7 * K)
    W = inputs.normal_bf16((N, K), 0.02, seed=N + 1)
    wq, wsc = orc.quantize_rows_e4m3(W)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    xv = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    xm = torch.empty(sp24.meta_bytes(M, K), dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sp24.prune_compress_activations_fused_e4m3(dev_bf16(X), dev(wq), dev(wsc), Y, x_values=xv, x_meta=xm,
                                               x_scales=xs)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    ref = OracleSparseW(X, e4m3=True)  # the oracle's prune + per-row e4m3 cast, applied to X's rows
    assert np.array_equal(u8(xv), ref.values)
    assert np.array_equal(u8(xm), ref.image)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), ref.scales.view(np.uint32))
    W_hat = orc.e4m3_decode(wq) * wsc.astype(np.float64)[:, None]
    y_ref, a_ref = orc.gemm_f64(ref.W_hat, W_hat)
    check_tolerance(Y.cpu().numpy().astype(np.float64), y_ref, a_ref, "activations e4m3 M%d N%d K%d" % (M, N, K))
    # workspace variant, bf16 output
    ws = torch.empty(sp24.activations_e4m3_workspace_bytes(M, K), dtype=torch.uint8, device="cuda")
    Y2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sp24.prune_compress_activations_fused_e4m3(dev_bf16(X), dev(wq), dev(wsc), Y2, workspace=ws)
    torch.cuda.synchronize()
    check_tolerance(Y2.float().cpu().numpy().astype(np.float64), y_ref, a_ref, "activations e4m3 ws")


@pytest.mark.parametrize("M,N,K", [(512, 384, 512), (300, 256, 1024)])
def test_activation_fused_pair_kernel(M, N, K):
    test_activation_fused_parity(M, N, K)


# ---------------------------------------------------------------------------
# 2:4 energy loss (diagnostic next to the prune)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("rows,K,dist", [(1, 256, "normal"), (200, 1024, "student"), (5120, 5120, "normal"),
                                         (37, 4096, "student")])
def test_energy_loss_matches_oracle(rows, K, dist):
    if dist == "normal":
        W = inputs.normal_bf16((rows, K), 0.02, seed=rows + K)
    else:
        W = inputs.student_t_bf16((rows, K), 3.0, seed=rows + K)
    W[0, : min(K, 64)] = 0  # a stretch of zeros (kept zeros)
    share = torch.empty(rows, dtype=torch.float64, device="cuda")
    sums = torch.full((2,), 7.0, dtype=torch.float64, device="cuda")  # the call zeroes it
    sp24.energy_loss(dev_bf16(W), share, sums)
    torch.cuda.synchronize()
    d, t, sh, e = orc.energy_loss(W)
    assert np.allclose(share.cpu().numpy(), sh, rtol=1e-12, atol=1e-15)
    s = sums.cpu().numpy()
    assert s[0] == pytest.approx(d.sum(), rel=1e-12) and s[1] == pytest.approx(t.sum(), rel=1e-12)
    assert s[0] / s[1] == pytest.approx(e, rel=1e-12)


def test_energy_loss_zero_rows():
    W = np.zeros((3, 64), np.uint16)
    share = torch.full((3,), 5.0, dtype=torch.float64, device="cuda")
    sp24.energy_loss(dev_bf16(W), share, None)
    torch.cuda.synchronize()
    assert share.cpu().numpy().tolist() == [0.0, 0.0, 0.0]


# ---------------------------------------------------------------------------
# full-size configurations, sampled outputs
# ---------------------------------------------------------------------------

def _sampled_check(X_hat_rows, W_hat_rows, y_gpu, ms, ns, what):
    y_ref, a_ref = orc.gemm_f64_sampled(X_hat_rows, W_hat_rows, ms, ns)
    check_tolerance(y_gpu[ms, ns], y_ref, a_ref, what)


@pytest.mark.parametrize("N,K", inputs.DECODE_NK)
def test_decode_full_size_sampled(N, K):
    M = 8
    X, W = inputs.linear_pair(M, N, K, seed=N + K)
    Wd = dev_bf16(W)
    vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    ws_ = torch.empty(N, dtype=torch.float32, device="cuda")
    sp24.prune_compress(Wd, sp24.E4M3, vals, meta, row_scales=ws_)
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sp24.quantize_e4m3_rows(dev_bf16(X), xq, xs)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.gemm_args(xq, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=ws_)
    ws = workspace_for(a)
    sp24.set_workspace(a, ws)
    sp24.gemm(a)
    torch.cuda.synchronize()
    g = np.random.default_rng(1)
    ns = g.choice(N, size=64, replace=False)
    ms = g.integers(0, M, size=64)
    # oracle on the sampled rows only
    ref = OracleSparseW(W[ns], e4m3=True)
    _, _, X_hat = oracle_x(X, True)
    y_ref, a_ref = orc.gemm_f64_sampled(X_hat, ref.W_hat, ms, np.arange(ns.size))
    y_gpu = Y.float().cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y_gpu, y_ref, a_ref, "decode %dx%d" % (N, K))


@pytest.mark.parametrize("e4", [False, True])
def test_prefill_full_size_sampled(e4):
    M, N, K = 2048, 4096, 4096
    X, W = inputs.linear_pair(M, N, K, seed=123, outliers=True)
    Wd = dev_bf16(W)
    vals = torch.empty(N, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    ws_ = torch.empty(N, dtype=torch.float32, device="cuda")
    sp24.prune_compress(Wd, sp24.E4M3 if e4 else sp24.BF16, vals, meta, row_scales=ws_ if e4 else None)
    if e4:
        Xd = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        xs = torch.empty(M, dtype=torch.float32, device="cuda")
        sp24.quantize_e4m3_rows(dev_bf16(X), Xd, xs)
    else:
        Xd, xs = dev_bf16(X), None
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.gemm_args(Xd, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs,
                       w_scales=ws_ if e4 else None)
    sp24.gemm(a)
    torch.cuda.synchronize()
    g = np.random.default_rng(2)
    ns = g.choice(N, size=48, replace=False)
    ms = g.integers(0, M, size=48)
    ref = OracleSparseW(W[ns], e4m3=e4)
    xq, xsc, X_hat = oracle_x(X[ms], e4)
    y_ref, a_ref = orc.gemm_f64_sampled(X_hat, ref.W_hat, np.arange(48), np.arange(48))
    y_gpu = Y.float().cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y_gpu, y_ref, a_ref, "prefill e4=%s" % e4)


@pytest.mark.parametrize("M,N,K", [(16384, 12288, 4096), (8192, 4096, 12288)])
@pytest.mark.parametrize("e4", [False, True])
def test_prefill_largest_shapes_full_size_sampled(M, N, K, e4):
    """The largest prefill shapes (many 256 x 256 tiles per CTA pair, K up to
    12288) on device-pruned weights with outliers; sampled outputs against the
    oracle."""
    X, W = inputs.linear_pair(M, N, K, seed=M + K, outliers=True)
    a, Y, _, _ = _prepare_large(X, W, e4, sp24.SPARSE)
    sp24.gemm(a)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    g = np.random.default_rng(M + N)
    ms = np.concatenate([g.integers(0, M, size=40), [0, M - 1]])
    ns = np.concatenate([g.integers(0, N, size=40), [0, N - 1]])
    W_hat = OracleSparseW(W[ns], e4m3=e4).W_hat
    _, _, X_hat = oracle_x(X[ms], e4)
    y_ref, a_ref = orc.gemm_f64_sampled(X_hat, W_hat, np.arange(ms.size), np.arange(ns.size))
    y_gpu = Y.float().cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y_gpu, y_ref, a_ref, "prefill M%d N%d K%d e4=%s" % (M, N, K, e4))


def test_tiny_configuration_seed0_matches_oracle():
    """The tiny configuration exactly as specified (X[16 x 256] ~ N(0,1),
    W[256 x 256] ~ N(0, 0.02^2), seed 0): W pruned and compressed on the
    device (values and metadata bit-exact to the oracle), then Y = X W^T with
    fp32 accumulation, bf16 and e4m3, within tolerance of the fp64 oracle."""
    X, W = inputs.tiny(0)
    M, K = X.shape
    N = W.shape[0]
    vals = torch.empty(N, K // 2, dtype=torch.bfloat16, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    sp24.prune_compress(dev_bf16(W), sp24.BF16, vals, meta)
    pruned, values, canon = orc.prune_compress_bf16(W)
    assert np.array_equal(bits16(vals), values)
    assert np.array_equal(u8(meta), orc.meta_image(canon, N, K, False))
    assert (values.reshape(N, K // 2).shape == (256, 128))
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    sp24.gemm(sp24.gemm_args(dev_bf16(X), vals, Y, K, sp24.SPARSE, W_meta=meta))
    torch.cuda.synchronize()
    y_ref, a_ref = orc.gemm_f64(orc.bf16_bits_to_f64(X), orc.bf16_bits_to_f64(pruned))
    check_tolerance(Y.cpu().numpy().astype(np.float64), y_ref, a_ref, "tiny bf16")
    y, y_ref, a_ref, _, _ = run_gemm(X, W, True, sp24.SPARSE, True)
    check_tolerance(y, y_ref, a_ref, "tiny e4m3")


@pytest.mark.parametrize("grouping", ["one_launch", "by_class"])
def test_decode_step_full_size_grouped_sampled(grouping):
    """The decode step as the benchmark times it: 16 GEMMs (M in 1, 8, 32, 128
    times the four weight shapes, e4m3 2:4 weights), one grouped per-token cast,
    then the 16 GEMMs as one grouped launch (each problem with its own
    token-tile width), or as one launch per token-count class with the second
    and third chained after the first as independent launches; weights marked
    static.  Sampled outputs of every GEMM against the oracle."""
    g = np.random.default_rng(7)
    Wb = {}
    for (N, K) in inputs.DECODE_NK:
        W = inputs.normal_bf16((N, K), 0.02, seed=N + K)
        vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
        meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
        sc = torch.empty(N, dtype=torch.float32, device="cuda")
        sp24.prune_compress(dev_bf16(W), sp24.E4M3, vals, meta, row_scales=sc)
        Wb[(N, K)] = (W, vals, meta, sc)
    items = []
    for M in inputs.DECODE_M:
        for i, (N, K) in enumerate(inputs.DECODE_NK):
            X = inputs.normal_bf16((M, K), 1.0, seed=M * 10 + i)
            xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
            xs = torch.empty(M, dtype=torch.float32, device="cuda")
            Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            _, vals, meta, sc = Wb[(N, K)]
            a = sp24.gemm_args(xq, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=sc,
                               flags=sp24.GEMM_W_STATIC)
            items.append(dict(M=M, N=N, K=K, X=X, Xd=dev_bf16(X), xq=xq, xs=xs, Y=Y, a=a))
    cast = sp24.QuantGroup([(it["Xd"], it["xq"], it["xs"]) for it in items])
    by = {}
    for it in items:
        by.setdefault(sp24.m_class(it["M"]) if grouping == "by_class" else 0, []).append(it["a"])
    groups = [sp24.GemmGroup(v, after_independent=i > 0) for i, (_, v) in enumerate(sorted(by.items()))]
    assert len(groups) == (3 if grouping == "by_class" else 1)
    torch.cuda.synchronize()
    for _ in range(2):  # the second pass runs on workspaces the first left at zero
        cast()
        for grp in groups:
            grp()
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    for it in items:
        M, N, K = it["M"], it["N"], it["K"]
        ns = g.choice(N, size=24, replace=False)
        ms = g.integers(0, M, size=24)
        ref = OracleSparseW(Wb[(N, K)][0][ns], e4m3=True)
        _, _, X_hat = oracle_x(it["X"], True)
        y_ref, a_ref = orc.gemm_f64_sampled(X_hat, ref.W_hat, ms, np.arange(ns.size))
        y_gpu = it["Y"].float().cpu().numpy().astype(np.float64)[ms, ns]
        check_tolerance(y_gpu, y_ref, a_ref, "decode step M%d %dx%d" % (M, N, K))


@pytest.mark.parametrize("name,M", [("gate_up", 4096), ("qkv", 16), ("o", 1), ("o", 256), ("down", 1),
                                    ("down", 256)])
def test_hybrid_full_size_sampled(name, M):
    """Hybrid weights (25% dense 128 x 128 tiles, e4m3) at full size: gate_up at
    4096 tokens runs on CTA pairs, qkv at 16 tokens on single CTAs.  The
    weights are pruned on the device; the oracle checks two whole 128-row
    blocks (their tile flags carried along) against 16 sampled tokens."""
    N, K = {n: (N_, K_) for n, N_, K_ in inputs.HYBRID_NK}[name]
    W = inputs.normal_bf16((N, K), 0.02, seed=N + 3)
    X = inputs.normal_bf16((M, K), 1.0, seed=M + 3)
    mask = inputs.hybrid_mask(N, K, seed=5)
    vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    dense = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    sc = torch.empty(N, dtype=torch.float32, device="cuda")
    sp24.prune_compress(dev_bf16(W), sp24.E4M3, vals, meta, row_scales=sc, tile_mask=dev(mask), dense_tiles=dense)
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sp24.quantize_e4m3_rows(dev_bf16(X), xq, xs)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.gemm_args(xq, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=sc,
                       tile_mask=dev(mask), W_dense_tiles=dense)
    sp24.set_workspace(a, workspace_for(a))
    sp24.gemm(a)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    g = np.random.default_rng(11)
    rbs = np.sort(g.choice(N // 128, size=2, replace=False))
    rows = np.concatenate([np.arange(128 * rb, 128 * rb + 128) for rb in rbs])
    ref = OracleSparseW(W[rows], e4m3=True, mask=mask[rbs])
    ms = np.sort(g.choice(M, size=min(M, 16), replace=False))
    _, _, X_hat = oracle_x(X[ms], True)
    y_ref, a_ref = orc.gemm_f64(X_hat, ref.W_hat)
    y_gpu = Y.float().cpu().numpy().astype(np.float64)[np.ix_(ms, rows)]
    check_tolerance(y_gpu, y_ref, a_ref, "hybrid %s M%d" % (name, M))


@pytest.mark.parametrize("e4", [False, True])
def test_activation_full_size_sampled(e4):
    """The online activation path at its full size (X 8192 x 4096 Student-t,
    W 12288 x 4096): compressed X of sampled rows and of the first row block's
    metadata bit-exact, sampled outputs within tolerance."""
    M, K, N = inputs.ACT_SHAPE["M"], inputs.ACT_SHAPE["K"], inputs.ACT_SHAPE["N"]
    X = inputs.student_t_bf16((M, K), 3.0, seed=4)
    W = inputs.normal_bf16((N, K), 0.02, seed=4)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    xm = torch.empty(sp24.meta_bytes(M, K), dtype=torch.uint8, device="cuda")
    xv = torch.empty(M, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device="cuda")
    if e4:
        wq, wsc = orc.quantize_rows_e4m3(W)
        xs = torch.empty(M, dtype=torch.float32, device="cuda")
        sp24.prune_compress_activations_fused_e4m3(dev_bf16(X), dev(wq), dev(wsc), Y, x_values=xv, x_meta=xm,
                                                   x_scales=xs)
    else:
        sp24.prune_compress_activations_fused(dev_bf16(X), dev_bf16(W), Y, x_values=xv, x_meta=xm)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    g = np.random.default_rng(13)
    ms = np.sort(g.choice(M, size=32, replace=False))
    ns = np.sort(g.choice(N, size=32, replace=False))
    img0 = u8(xm)[:(K // 128) * 2048]  # row block 0's chunks come first in the image
    if e4:
        ref = OracleSparseW(X[ms], e4m3=True)
        assert np.array_equal(u8(xv)[ms], ref.values)
        assert np.array_equal(xs.cpu().numpy()[ms].view(np.uint32), ref.scales.view(np.uint32))
        assert np.array_equal(img0, OracleSparseW(X[:128], e4m3=True).image)
        W_hat = orc.e4m3_decode(wq[ns]) * wsc[ns].astype(np.float64)[:, None]
        X_hat = ref.W_hat
    else:
        pruned, vals, canon = orc.prune_compress_bf16(X[ms])
        assert np.array_equal(bits16(xv)[ms], vals)
        _, _, canon0 = orc.prune_compress_bf16(X[:128])
        assert np.array_equal(img0, orc.meta_image(canon0, 128, K, False))
        W_hat = orc.bf16_bits_to_f64(W[ns])
        X_hat = orc.bf16_bits_to_f64(pruned)
    y_ref, a_ref = orc.gemm_f64(X_hat, W_hat)
    y_gpu = Y.float().cpu().numpy().astype(np.float64)[np.ix_(ms, ns)]
    check_tolerance(y_gpu, y_ref, a_ref, "activations full size e4=%s" % e4)


# ---------------------------------------------------------------------------
# tactic selector (kernel 5) and the bounded wait
# ---------------------------------------------------------------------------

def test_select_tactic_record():
    M, N, K = 8, 1024, 4096
    X, W = inputs.linear_pair(M, N, K, seed=4)
    _, _, _, sa, ws = run_gemm(X, W, True, sp24.SPARSE, False)
    _, _, _, da, _ = run_gemm(X, W, True, sp24.DENSE, False)
    rec = sp24.select_tactic(sa, da, warmup=2, iters=9)
    assert rec["eligible"] and rec["iters"] == 9
    assert rec["t_sparse_us"] > 0 and rec["t_dense_us"] > 0
    assert rec["t_sparse_min_us"] <= rec["t_sparse_us"]
    expect = orc.select_tactic([rec["t_sparse_us"]], [rec["t_dense_us"]])[0]
    assert rec["selected"] == expect
    assert (rec["reason"] == "") == (expect == "sparse")
    # an ineligible sparse call (N not a multiple of 128) falls back to dense
    sa.N = 1000
    rec2 = sp24.select_tactic(sa, da, warmup=1, iters=3)
    assert not rec2["eligible"] and rec2["selected"] == "dense" and rec2["reason"] == "Alignment failure"


def test_bounded_wait_expires_without_fault_and_context_survives():
    sp24.clear_device_error()
    assert sp24.selftest_bounded_wait(2_000_000) == sp24.SP24_ERR_DEVICE_TIMEOUT
    assert sp24.last_device_error() == sp24.SP24_ERR_DEVICE_TIMEOUT
    assert sp24.clear_device_error() == sp24.SP24_OK
    assert sp24.last_device_error() == sp24.SP24_OK
    # the context is still usable
    X, W = inputs.linear_pair(16, 256, 256, seed=0)
    y, y_ref, a_ref, _, _ = run_gemm(X, W, False, sp24.SPARSE, True)
    check_tolerance(y, y_ref, a_ref, "after self test")


# ---------------------------------------------------------------------------
# online activations pruned inside the GEMM (no compressed X in HBM)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (300, 384, 640), (512, 768, 1024), (1024, 512, 4096),
                                   (260, 1280, 256)])
def test_prune_in_gemm_parity(M, N, K):
    X = inputs.student_t_bf16((M, K), 3.0, seed=M + 5 * K)
    X[3, :8] = np.array([0x3F80, 0xBF80, 0x3F80, 0, 0, 0, 0, 0], np.uint16)  # ties, zero group
    W = inputs.normal_bf16((N, K), 0.02, seed=N + 9)
    pruned, values, canon = orc.prune_compress_bf16(X)
    y_ref, a_ref = orc.gemm_f64(orc.bf16_bits_to_f64(pruned), orc.bf16_bits_to_f64(W))
    Xd, Wd = dev_bf16(X), dev_bf16(W)
    for emit in (False, True):
        for out_f32 in (True, False):
            Y = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
            Y.fill_(float("nan"))
            xv = torch.empty(M, K // 2, dtype=torch.bfloat16, device="cuda") if emit else None
            xm = torch.empty(sp24.meta_bytes(M, K), dtype=torch.uint8, device="cuda") if emit else None
            sp24.prune_activations_in_gemm(Xd, Wd, Y, x_values=xv, x_meta=xm)
            torch.cuda.synchronize()
            assert sp24.last_device_error() == sp24.SP24_OK
            check_tolerance(Y.float().cpu().numpy().astype(np.float64), y_ref, a_ref,
                            "prune in gemm M%d N%d K%d f32=%s" % (M, N, K, out_f32))
            if emit:
                assert np.array_equal(bits16(xv), values), "emitted compressed X"
                assert np.array_equal(u8(xm), orc.meta_image(canon, M, K, False)), "emitted metadata image"


def test_prune_in_gemm_full_size_sampled():
    """cfg 4 at full size (X 8192 x 4096 Student-t, W 12288 x 4096): sampled
    outputs against the oracle and against the two-kernel path."""
    M, K, N = inputs.ACT_SHAPE["M"], inputs.ACT_SHAPE["K"], inputs.ACT_SHAPE["N"]
    X = inputs.student_t_bf16((M, K), 3.0, seed=4)
    W = inputs.normal_bf16((N, K), 0.02, seed=4)
    Xd, Wd = dev_bf16(X), dev_bf16(W)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sp24.prune_activations_in_gemm(Xd, Wd, Y)
    Y2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sp24.activations_workspace_bytes(M, K), dtype=torch.uint8, device="cuda")
    sp24.prune_compress_activations_fused(Xd, Wd, Y2, workspace=ws)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    g = np.random.default_rng(21)
    ms = np.concatenate([g.integers(0, M, size=60), [0, M - 1]])
    ns = np.concatenate([g.integers(0, N, size=60), [0, N - 1]])
    pruned, _, _ = orc.prune_compress_bf16(X[ms])
    y_ref, a_ref = orc.gemm_f64_sampled(orc.bf16_bits_to_f64(pruned), orc.bf16_bits_to_f64(W[ns]),
                                        np.arange(ms.size), np.arange(ns.size))
    y = Y.float().cpu().numpy().astype(np.float64)[ms, ns]
    y2 = Y2.float().cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y, y_ref, a_ref, "prune in gemm, full size")
    check_tolerance(y, y2, a_ref, "prune in gemm vs two-kernel path")
