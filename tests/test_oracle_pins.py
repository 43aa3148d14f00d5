"""Pins of the fp64 oracle to values and identities fixed by the pages and by
mathematics, independent of the oracle's own code.  CPU only."""
import math

import numpy as np
import pytest
import torch

import inputs
import oracle
from conftest import golden

DEF = inputs.DEFAULT_PENALTY


# ---------------------------------------------------------------- penalty --

def test_penalty_worked_table():
    """Flash Partitions page, section 3 table: penalty, factor, baseline, correction."""
    for dt, pen, factor, baseline, corr in golden("penalty_table.txt"):
        p = oracle.penalty(dt, *DEF)
        assert abs(p - pen) <= 0.005 + 1e-12, (dt, p, pen)
        assert abs(math.exp(-p) - factor) <= 5e-7
        assert abs(math.exp(-DEF[3]) - baseline) <= 5e-7
        assert abs((math.exp(-p) - math.exp(-DEF[3])) - corr) <= 5e-7 + 1e-12


def test_penalty_saturation_threshold():
    """Correction vanishes at window + falloff*sqrt(cap/strength) (~0.633 s); zero inside the window."""
    (strength, window, falloff, cap, printed, decimals), = golden("saturation.txt")
    thr = window + falloff * math.sqrt(cap / strength)
    assert abs(thr - printed) <= 0.5 * 10 ** -int(decimals)
    for dt in np.linspace(0.0, window, 11):
        assert oracle.penalty(dt, strength, window, falloff, cap) == 0.0
    for dt in [thr + 1e-9, thr + 0.01, 0.8, 1.5, 10.0]:
        p = oracle.penalty(dt, strength, window, falloff, cap)
        assert p == cap and math.exp(-p) - math.exp(-cap) == 0.0
    for dt in [window + 1e-6, 0.3, 0.5, thr - 1e-6]:
        p = oracle.penalty(dt, strength, window, falloff, cap)
        assert 0.0 < p < cap and math.exp(-p) - math.exp(-cap) > 0.0


def test_penalty_monotone_bounded_and_reductions():
    dts = np.linspace(0, 3, 3001)
    ps = [oracle.penalty(t, *DEF) for t in dts]
    assert all(0.0 <= p <= DEF[3] for p in ps)
    assert all(b >= a for a, b in zip(ps, ps[1:]))
    # strength = 0 or cap = 0 removes the penalty (Flash Partitions page, section 4 end)
    assert all(oracle.penalty(t, 0.0, 0.2, 0.25, 6.0) == 0.0 for t in dts)
    assert all(oracle.penalty(t, 2.0, 0.2, 0.25, 0.0) == 0.0 for t in dts)


def test_decomposition_identity():
    """exp(-p) = exp(-cap) + [exp(-p) - exp(-cap)], both terms >= 0 (section 3)."""
    cap = DEF[3]
    for t in np.linspace(0, 2, 401):
        p = oracle.penalty(t, *DEF)
        base, corr = math.exp(-cap), math.exp(-p) - math.exp(-cap)
        assert base > 0 and corr >= 0
        assert abs(base + corr - math.exp(-p)) <= 1e-15


# ------------------------------------------------------------- helpers --

def _tiny(seed=7, frames=6, gtok=20, otok=22, text=20, audio=30, H=2, d=32, cluster=0.0):
    segs = [inputs.Segment(inputs.SEG_TEXT, text), inputs.Segment(inputs.SEG_AUDIO, audio),
            inputs.Segment(inputs.SEG_GUIDE, frames * gtok, frames),
            inputs.Segment(inputs.SEG_OUTPUT, frames * otok, frames)]
    cfg = inputs.custom(H, d, segs, seed, cluster_norm=cluster, penalty=DEF)
    seg, times, _ = cfg.layout()
    q = inputs.tensor(cfg, inputs.TENSOR_Q)
    k = inputs.tensor(cfg, inputs.TENSOR_K)
    v = inputs.tensor(cfg, inputs.TENSOR_V)
    return cfg, seg, times, q, k, v


def _f64(x):
    return torch.from_numpy(inputs.bf16_bits_to_f64(x))


def _sdpa(q, k, v, mask=None):
    """torch's scaled_dot_product_attention in fp64 on CPU (library routine)."""
    return torch.nn.functional.scaled_dot_product_attention(
        _f64(q)[None], _f64(k)[None], _f64(v)[None], attn_mask=mask).numpy()[0]


def _bias(seg, times, pen):
    """-penalty on output-query x guide-key pairs (edge rule of the Flash Partitions page, section 1)."""
    S = len(seg)
    b = np.zeros((S, S))
    qi = np.where(seg == inputs.SEG_OUTPUT)[0]
    kj = np.where(seg == inputs.SEG_GUIDE)[0]
    for i in qi:
        for j in kj:
            b[i, j] = -oracle.penalty(abs(float(times[i]) - float(times[j])), *pen)
    return torch.from_numpy(b)


# ------------------------------------------------------------ attention --

@pytest.mark.parametrize("pen", [None, (0.0, 0.2, 0.25, 6.0), (2.0, 0.2, 0.25, 0.0)])
def test_unbiased_reduces_to_library_softmax(pen):
    """No penalty, strength 0 or cap 0 -> textbook softmax(QK^T/sqrt(d))V (torch SDPA, fp64)."""
    cfg, seg, times, q, k, v = _tiny()
    o, lse = oracle.attend(q, k, v, seg, times, pen=pen)
    ref = _sdpa(q, k, v)
    H, S, d = q.shape
    assert np.abs(o.reshape(H, S, d) - ref).max() < 1e-12
    s = torch.einsum("hid,hjd->hij", _f64(q), _f64(k)) / math.sqrt(d)
    assert np.abs(lse.reshape(H, S) - torch.logsumexp(s, -1).numpy()).max() < 1e-12


@pytest.mark.parametrize("pen", [DEF, (0.5, 0.1, 0.3, 3.0), (8.0, 0.2, 0.25, 12.0)])
def test_biased_matches_library_with_explicit_bias(pen):
    """Penalty on output->guide edges only == SDPA with the explicit additive bias."""
    cfg, seg, times, q, k, v = _tiny()
    o, lse = oracle.attend(q, k, v, seg, times, pen=pen)
    bias = _bias(seg, times, pen)
    ref = _sdpa(q, k, v, mask=bias)
    H, S, d = q.shape
    assert np.abs(o.reshape(H, S, d) - ref).max() < 1e-12
    s = torch.einsum("hid,hjd->hij", _f64(q), _f64(k)) / math.sqrt(d) + bias
    assert np.abs(lse.reshape(H, S) - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def test_bias_changes_only_output_rows():
    cfg, seg, times, q, k, v = _tiny()
    o0, _ = oracle.attend(q, k, v, seg, times, pen=None)
    o1, _ = oracle.attend(q, k, v, seg, times, pen=DEF)
    H, S, d = q.shape
    diff = np.abs(o1 - o0).reshape(H, S, d).max(axis=(0, 2))
    assert np.all(diff[seg != inputs.SEG_OUTPUT] == 0.0)
    assert np.all(diff[seg == inputs.SEG_OUTPUT] > 0.0)


@pytest.mark.parametrize("pen", [DEF, (0.5, 0.1, 0.3, 3.0), (8.0, 0.2, 0.25, 12.0),
                                 (2.0, 0.0, 0.25, 1.0), (2.0, 0.2, 0.05, 6.0)])
@pytest.mark.parametrize("layout", [dict(), dict(frames=9, gtok=13, otok=11),
                                    dict(frames=4, gtok=33, otok=31, text=7, audio=5)])
def test_partition_merge_equals_direct(pen, layout):
    """Flash-Partitions decomposition + log-sum-exp merge (sections 3-4) equals the direct
    rule at several strengths/caps and frame layouts (frames straddle 16-row blocks)."""
    cfg, seg, times, q, k, v = _tiny(**layout)
    o1, l1 = oracle.attend(q, k, v, seg, times, pen=pen, B=16)
    o2, l2 = oracle.attend_partitions(q, k, v, seg, times, pen=pen, B=16)
    assert np.abs(o1 - o2).max() < 1e-12
    assert np.abs(l1 - l2).max() < 1e-12


def test_output_is_convex_combination():
    cfg, seg, times, q, k, v = _tiny()
    o, _ = oracle.attend(q, k, v, seg, times, pen=DEF)
    H, S, d = q.shape
    vf = inputs.bf16_bits_to_f64(v)
    o = o.reshape(H, S, d)
    assert np.all(o <= vf.max(axis=1, keepdims=True) + 1e-12)
    assert np.all(o >= vf.min(axis=1, keepdims=True) - 1e-12)


# -------------------------------------------------------------- routing --

def _route_case(seed=11, H=3, d=32, frames=8, tok=48):
    segs = [inputs.Segment(inputs.SEG_TEXT, 40), inputs.Segment(inputs.SEG_AUDIO, 50),
            inputs.Segment(inputs.SEG_OUTPUT, frames * tok, frames)]
    cfg = inputs.custom(H, d, segs, seed, cluster_norm=2.0)
    seg, times, _ = cfg.layout()
    return cfg, seg, times, inputs.tensor(cfg, 0), inputs.tensor(cfg, 1), inputs.tensor(cfg, 2)


def test_pool_is_block_mean():
    cfg, seg, times, q, k, v = _route_case()
    B = 16
    p = oracle.pool(q, B)
    x = inputs.bf16_bits_to_f64(q)
    H, S, d = x.shape
    for b in range(p.shape[1]):
        ref = x[:, b * B:min(S, (b + 1) * B)].mean(axis=1)
        assert np.abs(p[:, b] - ref).max() < 1e-14


def test_block_classes_and_k():
    seg = np.array([0] * 70 + [2] * 10 + [3] * 100 + [4] * 50, np.uint8)  # S = 230
    cls = oracle.block_classes(seg, 64)
    assert list(cls) == [1, 1, 0, 0]          # block 1 mixes audio rows 64..79 and video
    for nv in [1, 2, 7, 246, 741, 1794]:
        for s in [0.0, 0.6, 0.85, 0.9, 0.999]:
            kk = oracle.k_for(nv, s)
            assert 1 <= kk <= nv
            assert kk >= (1 - s) * nv - 1e-6 and (kk - 1 < (1 - s) * nv or kk == 1)
    assert oracle.k_for(1794, 0.90) == 180 and oracle.k_for(246, 0.85) == 37
    assert oracle.k_for(50, 0.0) == 50


@pytest.mark.parametrize("sparsity", [0.5, 0.75, 0.9])
def test_route_matches_library_topk(sparsity):
    """Pooled scores by torch (mean + matmul) and selection by torch.topk give the same sets."""
    cfg, seg, times, q, k, v = _route_case()
    B = 16
    sel, scores, kth = oracle.route(q, k, seg, sparsity, B=B, want_scores=True)
    cls = oracle.block_classes(seg, B)
    vid = np.where(cls == 0)[0]
    H, S, d = q.shape
    nkb = (S + B - 1) // B

    def pooled(x):
        x = _f64(x)
        return torch.stack([x[:, b * B:min(S, (b + 1) * B)].mean(1) for b in range(nkb)], 1)
    qp, kp = pooled(q)[:, vid], pooled(k)[:, vid]
    ref = torch.einsum("hid,hjd->hij", qp, kp) / math.sqrt(d)
    assert np.abs(scores - ref.numpy()).max() < 1e-12
    kk = sel.shape[-1]
    top = torch.topk(ref, kk, dim=-1).indices.numpy()
    for h in range(H):
        for i in range(len(vid)):
            assert sorted(vid[top[h, i]].tolist()) == sel[h, i].tolist()
            assert kth[h, i] == pytest.approx(float(torch.sort(ref[h, i], descending=True).values[kk - 1]), abs=1e-15)


def test_route_invariants_and_dense_limit():
    cfg, seg, times, q, k, v = _route_case()
    B = 16
    cls = oracle.block_classes(seg, B)
    vid = set(np.where(cls == 0)[0].tolist())
    sel, _, _ = oracle.route(q, k, seg, 0.8, B=B)
    for lst in sel.reshape(-1, sel.shape[-1]):
        assert list(lst) == sorted(set(lst.tolist())) and set(lst.tolist()) <= vid
    sel0, _, _ = oracle.route(q, k, seg, 0.0, B=B)
    assert np.all(sel0 == np.array(sorted(vid))[None, None, :])


def test_route_tie_goes_to_lower_block():
    """Two identical key blocks score exactly alike: the lower index must win."""
    cfg, seg, times, q, k, v = _route_case(H=1)
    B = 16
    cls = oracle.block_classes(seg, B)
    vid = np.where(cls == 0)[0]
    k = k.copy()
    a, b = int(vid[3]), int(vid[9])
    k[:, b * B:(b + 1) * B] = k[:, a * B:(a + 1) * B]
    nv = len(vid)
    sel, scores, kth = oracle.route(q, k, seg, 0.0, B=B, want_scores=True)
    for s in np.linspace(0.05, 0.95, 19):
        sel, scores, kth = oracle.route(q, k, seg, s, B=B, want_scores=True)
        for i in range(nv):
            row = sel[0, i].tolist()
            if (a in row) != (b in row):        # cut falls between the twins
                assert a in row and b not in row


def test_routed_attention_matches_masked_library_softmax():
    """Routed attention == SDPA with -inf on the key blocks a query block does not attend."""
    cfg, seg, times, q, k, v = _route_case(H=2, d=32, frames=6, tok=40)
    B = 16
    sel, _, _ = oracle.route(q, k, seg, 0.7, B=B)
    o, lse = oracle.attend(q, k, v, seg, times, pen=None, sel=sel, B=B)
    cls = oracle.block_classes(seg, B)
    vid_index = {b: i for i, b in enumerate(np.where(cls == 0)[0])}
    H, S, d = q.shape
    nkb = (S + B - 1) // B
    ref = np.empty((H, S, d))
    for h in range(H):
        mask = torch.zeros(S, S, dtype=torch.float64)
        for i in range(S):
            qb = i // B
            if cls[qb]:
                continue
            allowed = set(np.where(cls == 1)[0].tolist()) | set(sel[h, vid_index[qb]].tolist())
            for kb in range(nkb):
                if kb not in allowed:
                    mask[i, kb * B:(kb + 1) * B] = -math.inf
        ref[h] = torch.nn.functional.scaled_dot_product_attention(
            _f64(q)[h:h + 1], _f64(k)[h:h + 1], _f64(v)[h:h + 1], attn_mask=mask).numpy()[0]
    assert np.abs(o.reshape(H, S, d) - ref).max() < 1e-12
    # the partition path agrees on routed lists too
    o2, l2 = oracle.attend_partitions(q, k, v, seg, times, pen=DEF, sel=sel, B=B)
    o3, l3 = oracle.attend(q, k, v, seg, times, pen=DEF, sel=sel, B=B)
    assert np.abs(o2 - o3).max() < 1e-12 and np.abs(l2 - l3).max() < 1e-12


def test_sparsity_zero_equals_dense():
    cfg, seg, times, q, k, v = _route_case(H=2, frames=5, tok=40)
    B = 16
    sel, _, _ = oracle.route(q, k, seg, 0.0, B=B)
    o1, l1 = oracle.attend(q, k, v, seg, times, pen=DEF, sel=sel, B=B)
    o2, l2 = oracle.attend(q, k, v, seg, times, pen=DEF, sel=None, B=B)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_sampled_rows_equal_full_rows():
    cfg, seg, times, q, k, v = _tiny()
    H, S, d = q.shape
    o, lse = oracle.attend(q, k, v, seg, times, pen=DEF)
    heads = np.array([0, 1, 1, 0]); rows = np.array([0, S - 1, 100, 250])
    o2, l2 = oracle.attend(q, k, v, seg, times, pen=DEF, heads=heads, rows=rows)
    assert np.array_equal(o2, o.reshape(H, S, d)[heads, rows])
    assert np.array_equal(l2, lse.reshape(H, S)[heads, rows])


# ------------------------------------------------------------------ partition merge
# "Flash Partitions for H3 native temporal alignment", section 4: normalised partition outputs
# O_i with log normalisers L_i and multipliers w_i merge through logsumexp of L_i + log w_i.
# Pinned against brute-force softmax over disjoint key sets (numpy, fp64), not against the
# oracle's own partition path.

def _brute_partitions(x, v, groups, w=None):
    """x [rows][n_keys] scores, v [n_keys][d]; groups: disjoint key index lists.
    Returns per-group (O_g, L_g) and the weighted softmax over all keys."""
    parts_o, parts_l = [], []
    for g in groups:
        e = np.exp(x[:, g])
        parts_l.append(np.log(e.sum(axis=1)))
        parts_o.append(e @ v[g] / e.sum(axis=1, keepdims=True))
    mult = np.ones(x.shape[1])
    if w is not None:
        for g, wg in zip(groups, w):
            mult[g] = wg
    e = np.exp(x) * mult[None, :]
    return np.array(parts_o), np.array(parts_l), e @ v / e.sum(axis=1, keepdims=True), np.log(e.sum(axis=1))


def test_merge_of_disjoint_partitions_is_the_softmax_over_their_union():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 3, size=(7, 40))
    v = rng.normal(size=(40, 5))
    groups = [list(range(0, 9)), list(range(9, 30)), list(range(30, 40))]
    po, pl, want_o, want_l = _brute_partitions(x, v, groups)
    o, l = oracle.merge(po, pl)
    assert np.abs(o - want_o).max() < 1e-12 and np.abs(l - want_l).max() < 1e-12


def test_merge_weights_scale_each_partitions_probabilities():
    rng = np.random.default_rng(6)
    x = rng.normal(0, 2, size=(5, 24))
    v = rng.normal(size=(24, 3))
    groups = [list(range(0, 10)), list(range(10, 24))]
    w = [0.25, 1.7]
    po, pl, want_o, want_l = _brute_partitions(x, v, groups, w)
    o, l = oracle.merge(po, pl, np.log(w))
    assert np.abs(o - want_o).max() < 1e-12 and np.abs(l - want_l).max() < 1e-12


def test_merge_special_cases():
    rng = np.random.default_rng(7)
    po = rng.normal(size=(2, 4, 3))
    pl = rng.normal(size=(2, 4))
    o, l = oracle.merge(po[:1], pl[:1])                         # one partition, weight 1: unchanged
    assert np.array_equal(o, po[0]) and np.allclose(l, pl[0], atol=0, rtol=0)
    o, l = oracle.merge(po, pl, np.array([0.0, -np.inf]))       # weight 0 drops a partition
    assert np.allclose(o, po[0], atol=1e-15) and np.allclose(l, pl[0], atol=1e-15)
    o, l = oracle.merge(po, np.full((2, 4), -np.inf))           # nothing attended
    assert np.all(o == 0) and np.all(l == -np.inf)


# ------------------------------------------------------------------ pooled tail term
# "H3 SLA Attention", inputs table, tail_correction: the routed-out key blocks enter through one pooled
# term.  When every 64-row block consists of identical rows, a block's pooled score and mean value are
# exact for each of its rows, so routed attention with the tail term must equal dense attention.

def _blockwise_constant(cfg):
    """Q, K, V of cfg with every row replaced by its block's first row (bf16 bits)."""
    out = []
    for t in range(3):
        x = inputs.tensor(cfg, t).copy()
        H, S, d = x.shape
        for b in range(0, S, 64):
            x[:, b:b + 64] = x[:, b:b + 1]
        out.append(x)
    return out


def test_tail_term_is_exact_for_blockwise_constant_inputs():
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_AUDIO, 64),
            inputs.Segment(inputs.SEG_OUTPUT, 8 * 64, 8)]
    cfg = inputs.custom(2, 32, segs, seed=3, cluster_norm=2.0)
    seg, times, _ = cfg.layout()
    q, k, v = _blockwise_constant(cfg)
    sel, _, _ = oracle.route(q, k, seg, 0.75)
    H, S = 2, cfg.S
    heads, rows = np.repeat(np.arange(H), S), np.tile(np.arange(S), H)
    dense_o, dense_l = oracle.attend(q, k, v, seg, times, pen=None, sel=None, heads=heads, rows=rows)
    routed_o, _ = oracle.attend(q, k, v, seg, times, pen=None, sel=sel, heads=heads, rows=rows)
    tail_o, tail_l = oracle.attend_tail(q, k, v, seg, times, None, sel, heads, rows)
    assert np.abs(routed_o - dense_o).max() > 1e-3            # routing alone drops mass
    assert np.abs(tail_o - dense_o).max() < 1e-12 and np.abs(tail_l - dense_l).max() < 1e-12


def test_tail_term_weights_a_ragged_block_by_its_valid_rows():
    """The last video block holds 32 valid rows (S = 608): with blockwise-constant inputs the dense result
    counts that block's key 32 times, so the pooled term reproduces it only with the weight n_j = 32 (the
    valid rows), not the block size 64."""
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_AUDIO, 64),
            inputs.Segment(inputs.SEG_OUTPUT, 8 * 60, 8)]
    cfg = inputs.custom(2, 32, segs, seed=13, cluster_norm=2.0)
    seg, times, _ = cfg.layout()
    assert cfg.S == 608 and cfg.S % 64 == 32
    q, k, v = _blockwise_constant(cfg)
    sel, _, _ = oracle.route(q, k, seg, 0.75)
    last = cfg.S // 64
    assert np.any(np.all(sel != last, axis=-1))                  # some query blocks drop the ragged block
    H, S = 2, cfg.S
    heads, rows = np.repeat(np.arange(H), S), np.tile(np.arange(S), H)
    dense_o, dense_l = oracle.attend(q, k, v, seg, times, pen=None, sel=None, heads=heads, rows=rows)
    tail_o, tail_l = oracle.attend_tail(q, k, v, seg, times, None, sel, heads, rows)
    assert np.abs(tail_o - dense_o).max() < 1e-12 and np.abs(tail_l - dense_l).max() < 1e-12


def test_tail_term_is_absent_without_dropped_blocks():
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_OUTPUT, 4 * 64, 4)]
    cfg = inputs.custom(1, 32, segs, seed=4, cluster_norm=2.0)
    seg, times, _ = cfg.layout()
    q, k, v = (inputs.tensor(cfg, t) for t in range(3))
    sel, _, _ = oracle.route(q, k, seg, 0.0)                  # every video block kept
    lt, ot = oracle.tail(q, k, v, seg, sel)
    assert np.all(lt == -np.inf) and np.all(ot == 0)
    rows = np.arange(cfg.S)
    a = oracle.attend(q, k, v, seg, times, pen=None, sel=sel, heads=np.zeros_like(rows), rows=rows)
    b = oracle.attend_tail(q, k, v, seg, times, None, sel, np.zeros_like(rows), rows)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------- int8 QK --
# "H3 SLA Attention", inputs table, use_int8_qk: Q and K quantised per token
# with a dynamic scale before the QK dot product; PV unchanged.

def _bits(vals):
    return inputs.f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_quantize_hand_row():
    """max |x| = 1: scale 1/127, codes 127 x rounded half to even (63.5 -> 64, -63.5 -> -64)."""
    x = _bits([[1.0, -0.5, 0.25, 0.125, 0.75, -1.0, 0.0, 0.5]])
    codes, scales = oracle.quantize_rows(x)
    assert codes.tolist() == [[127, -64, 32, 16, 95, -127, 0, 64]]
    assert scales[0] == np.float32(1.0) / np.float32(127.0)


def _f32_from_exact(num, den):
    """The float32 nearest (ties to even) to (num / den) * 2^-149, for positive integers num, den with
    num / den < 2^23 (the subnormal range, whose spacing is 2^-149)."""
    from fractions import Fraction
    v = Fraction(num, den)
    n = v.numerator // v.denominator
    r = v - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.array([n], np.uint32).view(np.float32)[0]


def test_quantize_row_with_tiny_maximum():
    """Rows whose max |x| is far below 1 (reading of the per-token rule: quotients and products in fp32).
    Max 2^-120: 127/max = 127 * 2^120 is finite, so the codes are exact (half the max -> 63.5 -> 64).
    Max 2^-130 (a bf16 subnormal): 127/max overflows to +inf in fp32, so every nonzero element takes the
    code +-127 and zeros take 0 (0 * inf is NaN, read as 0).  The scales are max/127 rounded to fp32,
    here subnormal: computed exactly by hand."""
    x = np.zeros((2, 8), np.uint16)
    x[0, :4] = [0x0380, 0x0300, 0x8380, 0x0000]   # 2^-120, 2^-121, -2^-120, 0
    x[1, :4] = [0x0008, 0x8004, 0x0000, 0x0001]   # 2^-130, -2^-131, 0, 2^-133 (subnormal bf16)
    codes, scales = oracle.quantize_rows(x)
    assert codes[0].tolist() == [127, 64, -127, 0, 0, 0, 0, 0]
    assert codes[1].tolist() == [127, -127, 0, 127, 0, 0, 0, 0]
    assert scales[0] == _f32_from_exact(2 ** 29, 127)          # 2^-120 / 127 = 2^29 / 127 * 2^-149
    assert scales[1] == _f32_from_exact(2 ** 19, 127)          # 2^-130 / 127


def test_quantize_zero_row_and_power_of_two_invariance():
    x = np.zeros((1, 16), np.uint16)
    codes, scales = oracle.quantize_rows(x)
    assert not codes.any() and scales[0] == 0.0
    rng = np.random.default_rng(3)
    base = rng.standard_normal((5, 64)).astype(np.float32)
    c0, s0 = oracle.quantize_rows(_bits(base))
    for e in (-6, -1, 3, 9):
        c, s = oracle.quantize_rows(_bits(base * np.float32(2.0 ** e)))
        assert np.array_equal(c, c0)
        assert np.array_equal(s, s0 * np.float32(2.0 ** e))


def test_quantize_reconstruction_bound():
    """Every code is within half a step of x / s, and each nonzero row reaches +-127."""
    rng = np.random.default_rng(5)
    xb = _bits(rng.standard_normal((200, 128)) * rng.uniform(0.01, 30.0, (200, 1)))
    codes, scales = oracle.quantize_rows(xb)
    x = inputs.bf16_bits_to_f64(xb)
    err = np.abs(x - codes.astype(np.float64) * scales[:, None].astype(np.float64))
    assert np.all(err <= 0.5 * scales[:, None] * (1 + 1e-5))
    assert np.all(np.abs(codes).max(axis=1) == 127)


def _exact_int8_rows(rng, H, S, d):
    """bf16 rows code * 2^-7 with integer codes in [-127, 127] and one +-127 per row: the quantiser
    reproduces them exactly (scale 2^-7)."""
    c = rng.integers(-127, 128, (H, S, d))
    c[..., 0] = np.where(rng.random((H, S)) < 0.5, 127, -127)
    return _bits(c.astype(np.float32) / 128.0), c


def test_qk8_attend_equals_exact_on_exactly_quantisable_inputs():
    """When Q and K are exactly int8 times a per-row scale, the int8 score equals the exact one."""
    segs = [inputs.Segment(inputs.SEG_TEXT, 40), inputs.Segment(inputs.SEG_GUIDE, 3 * 30, 3),
            inputs.Segment(inputs.SEG_OUTPUT, 3 * 30, 3)]
    cfg = inputs.custom(2, 32, segs, seed=8)
    seg, times, _ = cfg.layout()
    rng = np.random.default_rng(9)
    q, cq = _exact_int8_rows(rng, cfg.H, cfg.S, 32)
    k, ck = _exact_int8_rows(rng, cfg.H, cfg.S, 32)
    v = inputs.tensor(cfg, 2)
    q8, sq = oracle.quantize_rows(q)
    assert np.array_equal(q8, cq) and np.all(sq == np.float32(2.0 ** -7))
    o8, l8 = oracle.attend_qk8(q, k, v, seg, times, pen=DEF)
    o, l = oracle.attend(q, k, v, seg, times, pen=DEF)
    assert np.abs(o8 - o).max() <= 1e-12 and np.abs(l8 - l).max() <= 1e-12


def test_qk8_attend_error_against_exact():
    """Gaussian Q/K/V: the int8 QK outputs stay within a few percent of the exact ones (the page reports
    about 1 % per layer for its int8 attention)."""
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_GUIDE, 4 * 48, 4),
            inputs.Segment(inputs.SEG_OUTPUT, 4 * 48, 4)]
    cfg = inputs.custom(2, 128, segs, seed=12, cluster_norm=2.0)
    seg, times, _ = cfg.layout()
    q, k, v = (inputs.tensor(cfg, i) for i in range(3))
    o8, _ = oracle.attend_qk8(q, k, v, seg, times, pen=DEF)
    o, _ = oracle.attend(q, k, v, seg, times, pen=DEF)
    rel = np.linalg.norm(o8 - o) / np.linalg.norm(o)
    assert 0.0 < rel <= 0.03, rel
