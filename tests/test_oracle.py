"""Pins for the fp64 oracle (CPU only).

Each test ties the oracle to something other than itself: numbers the pages
print, closed forms, invariants of the method, special cases that reduce to a
library routine (a single dot product, torch.topk, torch SDPA), and brute
force over all subsets on tiny inputs.  A dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import pytest
import torch

import oracle
from sparse_attention_04_b200 import inputs as dsa_inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _offsets(eps):
    o = [0]
    for e in eps:
        o.append(o[-1] + e)
    return torch.tensor(o, dtype=torch.int32)


# ---------------------------------------------------------------- decoders

def test_bf16_decoder_matches_torch_for_every_pattern():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64)
    for b in list(range(0, 1 << 16, 97)) + [0x0000, 0x8000, 0x3F80, 0xBF80, 0x7F7F, 0x0001]:
        want = ref[b].item()
        got = oracle.bf16_to_f64(b)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want)


def test_e4m3_decoder_matches_torch_for_every_code():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        want, got = ref[c].item(), oracle.e4m3_to_f64(c)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want
    assert oracle.e4m3_to_f64(0x7E) == 448.0 and oracle.e4m3_to_f64(0x01) == 2.0 ** -9


# ---------------------------------------------------------------- indexer

def _idx_case(E=40, T=1, B=1, seed=0):
    g = torch.Generator().manual_seed(seed)
    q = _bf16((B, T, 64, 128), seed + 1)
    k = _bf16((B * E, 128), seed + 2)
    w = torch.randn((B, T, 64), generator=g).float() * 0.01
    return q, w, k, _offsets([E] * B)


def test_indexer_one_hot_weight_is_relu_of_one_dot():
    """w = e_h reduces the score to ReLU(q_h . k_s): checks the head index and ReLU."""
    q, _, k, off = _idx_case(E=24)
    for h in (0, 17, 63):
        for sign in (1.0, -1.0):
            w = torch.zeros(1, 1, 64)
            w[0, 0, h] = sign
            sc = oracle.indexer_scores(q, w, k, None, off, 1, 1, 24)
            for s in range(24):
                dot = torch.dot(q[0, 0, h].double(), k[s].double()).item()
                assert sc[0, s].item() == pytest.approx(sign * max(dot, 0.0), rel=1e-12, abs=1e-12)


def test_indexer_sums_over_heads_and_is_linear_in_w():
    """The missing head sum was the bug fixed in the MLX port: I(w) = sum_h w_h I(e_h)."""
    q, w, k, off = _idx_case(E=16, seed=3)
    full = oracle.indexer_scores(q, w, k, None, off, 1, 1, 16)
    acc = torch.zeros(16, dtype=torch.float64)
    for h in range(64):
        e = torch.zeros(1, 1, 64)
        e[0, 0, h] = 1.0
        acc += w[0, 0, h].double() * oracle.indexer_scores(q, e, k, None, off, 1, 1, 16)[0]
    torch.testing.assert_close(full[0], acc, rtol=1e-12, atol=1e-12)


def test_indexer_zero_query_and_homogeneity():
    q, w, k, off = _idx_case(E=12, seed=5)
    z = oracle.indexer_scores(torch.zeros_like(q), w, k, None, off, 1, 1, 12)
    assert torch.all(z == 0)
    a = oracle.indexer_scores(q, w, k, None, off, 1, 1, 12)
    b = oracle.indexer_scores((q.float() * 2).to(torch.bfloat16), w, k, None, off, 1, 1, 12)
    torch.testing.assert_close(b, 2 * a, rtol=0, atol=0)


def test_indexer_causal_mask_and_ragged_offsets():
    """Prefill rows: s valid iff s <= start + t (start = E - T); -inf otherwise;
    nothing written at s >= E; sequences read their own cache slice."""
    eps, T = [9, 6], 4
    q = _bf16((2, T, 64, 128), 7)
    k = _bf16((sum(eps), 128), 8)
    w = torch.ones(2, T, 64)
    sc = oracle.indexer_scores(q, w, k, None, _offsets(eps), 2, T, 12)
    for b, E in enumerate(eps):
        for t in range(T):
            row = sc[b * T + t]
            t_abs = E - T + t
            for s in range(12):
                v = row[s].item()
                if s >= E:
                    assert math.isnan(v)
                elif s > t_abs:
                    assert v == -math.inf
                else:
                    base = sum(eps[:b])
                    want = sum(max(torch.dot(q[b, t, h].double(), k[base + s].double()).item(), 0.0)
                               for h in range(64))
                    assert v == pytest.approx(want, rel=1e-12)


def test_indexer_e4m3_equals_bf16_on_exactly_representable_codes():
    """Every e4m3 value is exact in bf16, so the e4m3 path with unit scales must equal
    the bf16 path on the decoded values, and k_scale must factor out of the sum."""
    g = torch.Generator().manual_seed(11)
    qc = torch.randint(0, 256, (1, 1, 64, 128), generator=g).to(torch.uint8)
    kc = torch.randint(0, 256, (20, 128), generator=g).to(torch.uint8)
    qc[(qc & 0x7F) == 0x7F] = 0  # drop the NaN code
    kc[(kc & 0x7F) == 0x7F] = 0
    w = torch.randn(1, 1, 64, generator=g) * 0.01
    off = _offsets([20])
    ones = torch.ones(20)
    e = oracle.indexer_scores(qc, w, kc, ones, off, 1, 1, 20)
    qb = qc.view(torch.float8_e4m3fn).to(torch.bfloat16)
    kb = kc.view(torch.float8_e4m3fn).to(torch.bfloat16)
    b = oracle.indexer_scores(qb, w, kb, None, off, 1, 1, 20)
    torch.testing.assert_close(e, b, rtol=0, atol=0)
    ks = torch.rand(20, generator=g) + 0.5
    e2 = oracle.indexer_scores(qc, w, kc, ks, off, 1, 1, 20)
    torch.testing.assert_close(e2[0], e[0] * ks.double(), rtol=1e-12, atol=1e-15)


def test_indexer_config_matches_page():
    cfg = json.load(open(os.path.join(GOLD, "indexer_config.json")))
    assert (dsa_inputs.H_I, dsa_inputs.D_I) == (cfg["index_n_heads"], cfg["index_head_dim"])
    assert dsa_inputs.WORKLOADS["decode32k"].topk == cfg["index_topk"]


# ---------------------------------------------------------------- top-k

def _brute_force_select(vals, valid, k):
    """The unique subset whose every member beats every valid non-member under
    (larger score, then lower position); found by trying all subsets."""
    cand = [s for s in range(len(vals)) if valid[s]]
    k_eff = min(k, len(cand))
    beats = lambda a, b: vals[a] > vals[b] or (vals[a] == vals[b] and a < b)
    found = [c for c in itertools.combinations(cand, k_eff)
             if all(beats(a, b) for a in c for b in cand if b not in c)]
    assert len(found) == 1
    return list(found[0]) + [-1] * (k - k_eff)


def test_topk_brute_force_all_subsets_with_ties():
    g = torch.Generator().manual_seed(2)
    alphabet = torch.tensor([-1.0, -0.0, 0.0, 0.5, 1.0], dtype=torch.float64)
    for trial in range(60):
        E = int(torch.randint(1, 10, (1,), generator=g))
        T = int(torch.randint(1, E + 1, (1,), generator=g))
        k = int(torch.randint(1, 6, (1,), generator=g))
        sc = alphabet[torch.randint(0, 5, (T, E), generator=g)]
        got = oracle.topk(sc, _offsets([E]), 1, T, k)
        for t in range(T):
            vals = [0.0 if v == 0 else v for v in sc[t].tolist()]
            valid = [s <= E - T + t for s in range(E)]
            assert got[t].tolist() == _brute_force_select(vals, valid, k)


def test_topk_matches_torch_topk_on_distinct_scores():
    g = torch.Generator().manual_seed(4)
    E, k = 3000, 2048
    sc = torch.randn(1, E, generator=g, dtype=torch.float64)
    got = oracle.topk(sc, _offsets([E]), 1, 1, k)[0]
    want = torch.sort(torch.topk(sc[0], k).indices).values.to(torch.int32)
    assert torch.equal(got, want)


def test_topk_maxtext_sizes_and_short_rows():
    """MaxText's reference test used index_topk=4, SEQ_LEN=8, and the review asked
    for SEQ_LEN < index_topk: rows with fewer valid positions keep all of them."""
    cfg = json.load(open(os.path.join(GOLD, "indexer_config.json")))
    k, L = cfg["test_index_topk"], cfg["test_seq_len"]
    g = torch.Generator().manual_seed(9)
    sc = torch.randn(L, L, generator=g, dtype=torch.float64)
    got = oracle.topk(sc, _offsets([L]), 1, L, k)
    for t in range(L):
        row = got[t].tolist()
        sel = [s for s in row if s >= 0]
        assert all(s <= t for s in sel)                 # masked positions never kept
        assert len(sel) == min(k, t + 1)
        if t + 1 <= k:
            assert sel == list(range(t + 1))
    got2 = oracle.topk(sc[:3, :3].contiguous(), _offsets([3]), 1, 3, 2 * k)
    assert got2[2].tolist() == [0, 1, 2] + [-1] * (2 * k - 3)


# ---------------------------------------------------------------- MLA

def _mla_case(E, T=1, H=4, seed=0):
    return _bf16((1, T, H, 576), seed + 1), _bf16((E, 576), seed + 2), _offsets([E])


def test_sparse_mla_equals_dense_when_all_positions_selected():
    """end_pos <= topk: the selection keeps every position, so sparse == dense
    (the MLX port skips the indexer in exactly this case)."""
    E, T, H = 37, 5, 3
    q, kv, off = _mla_case(E, T, H, seed=3)
    sc = torch.randn(T, E, dtype=torch.float64)
    idx = oracle.topk(sc, off, 1, T, 64)
    sp, lsp = oracle.sparse_mla(q, kv, off, idx, 1, T, H, 64, 0.07)
    de, lde = oracle.dense_mla(q, kv, off, 1, T, H, 0.07)
    torch.testing.assert_close(sp, de, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(lsp, lde, rtol=1e-12, atol=1e-12)


def test_dense_mla_matches_torch_sdpa():
    """MQA with K = row[:576] and V = row[:512], causal over start + t."""
    E, T, H, scale = 50, 6, 4, 576 ** -0.5
    q, kv, off = _mla_case(E, T, H, seed=5)
    out, lse = oracle.dense_mla(q, kv, off, 1, T, H, scale)
    Q = q[0].double().permute(1, 0, 2)                       # [H,T,576]
    K = kv.double()[None].expand(H, E, 576)
    V = kv.double()[:, :512][None].expand(H, E, 512)
    mask = torch.tensor([[s <= E - T + t for s in range(E)] for t in range(T)])
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=scale)
    torch.testing.assert_close(out, ref.permute(1, 0, 2), rtol=1e-10, atol=1e-12)
    logits = (Q @ K.transpose(-1, -2)) * scale
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1).permute(1, 0)
    torch.testing.assert_close(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_sparse_mla_closed_forms():
    E, H, k = 30, 5, 8
    q, kv, off = _mla_case(E, 1, H, seed=7)
    # one selected row: softmax weight 1, output = that row's first 512 values
    idx = torch.tensor([[13] + [-1] * (k - 1)], dtype=torch.int32)
    out, lse = oracle.sparse_mla(q, kv, off, idx, 1, 1, H, k, 0.1)
    for h in range(H):
        torch.testing.assert_close(out[0, h], kv[13, :512].double(), rtol=0, atol=1e-15)
        assert lse[0, h].item() == pytest.approx(0.1 * torch.dot(q[0, 0, h].double(), kv[13].double()).item(), rel=1e-12)
    # scale 0: uniform weights, output = mean of the selected rows
    sel = [2, 5, 11, 29]
    idx = torch.tensor([sel + [-1] * (k - 4)], dtype=torch.int32)
    out, lse = oracle.sparse_mla(q, kv, off, idx, 1, 1, H, k, 0.0)
    mean = kv[sel, :512].double().mean(0)
    for h in range(H):
        torch.testing.assert_close(out[0, h], mean, rtol=1e-12, atol=1e-14)
        assert lse[0, h].item() == pytest.approx(math.log(4), rel=1e-12)
    # the order of the index list does not matter; nothing selected -> zeros
    idx2 = torch.tensor([[29, -1, 5, -1, 11, 2, -1, -1]], dtype=torch.int32)
    out2, _ = oracle.sparse_mla(q, kv, off, idx2, 1, 1, H, k, 0.0)
    torch.testing.assert_close(out2, out, rtol=1e-13, atol=1e-15)
    none = torch.full((1, k), -1, dtype=torch.int32)
    out3, lse3 = oracle.sparse_mla(q, kv, off, none, 1, 1, H, k, 0.3)
    assert torch.all(out3 == 0) and torch.all(torch.isinf(lse3))


def _ragged_mla_case(eps, T, H, seed):
    """B = len(eps) sequences packed one after another in one cache, preceded
    by 3 rows no sequence owns (so a dropped base offset reads other rows)."""
    B = len(eps)
    q = _bf16((B, T, H, 576), seed + 1)
    pad = 3
    kv = _bf16((pad + sum(eps), 576), seed + 2)
    off = _offsets(eps) + pad
    return q, kv, off


def test_ragged_mla_sequences_use_their_own_cache_slice():
    """[Mask] decode listing: each sequence attends over its own kv_cache[:end_pos].
    With B = 3 ragged sequences in one cache, every row of sequence b must equal
    (1) the same oracle call on sequence b alone, with its slice of the cache as
    the whole cache, and (2) torch SDPA over that slice (sparse: the rows the
    index list names; dense: the causal prefix).  A missing or doubled base
    offset off[b] reads another sequence's rows and fails both."""
    eps, T, H, k, scale = [17, 40, 9], 2, 3, 12, 0.11
    B = len(eps)
    q, kv, off = _ragged_mla_case(eps, T, H, seed=21)
    g = torch.Generator().manual_seed(22)
    idx = torch.full((B * T, k), -1, dtype=torch.int32)
    for b, E in enumerate(eps):
        for t in range(T):
            n = min(k, E - 1)
            sel = torch.randperm(E, generator=g)[:n].to(torch.int32)
            idx[b * T + t, :n] = sel                      # unsorted, -1 holes at the end
    sp, lsp = oracle.sparse_mla(q, kv, off, idx, B, T, H, k, scale)
    de, lde = oracle.dense_mla(q, kv, off, B, T, H, scale)
    for b, E in enumerate(eps):
        lo = int(off[b])
        sl = kv[lo:lo + E].contiguous()
        one = _offsets([E])
        rows = slice(b * T, (b + 1) * T)
        sp1, lsp1 = oracle.sparse_mla(q[b:b + 1].contiguous(), sl, one, idx[rows].contiguous(), 1, T, H, k, scale)
        de1, lde1 = oracle.dense_mla(q[b:b + 1].contiguous(), sl, one, 1, T, H, scale)
        torch.testing.assert_close(sp[rows], sp1, rtol=0, atol=0)
        torch.testing.assert_close(lsp[rows], lsp1, rtol=0, atol=0)
        torch.testing.assert_close(de[rows], de1, rtol=0, atol=0)
        torch.testing.assert_close(lde[rows], lde1, rtol=0, atol=0)
        # torch SDPA over the slice: K = row[:576], V = row[:512]
        Q = q[b].double().permute(1, 0, 2)                # [H,T,576]
        K = sl.double()[None].expand(H, E, 576)
        V = sl.double()[:, :512][None].expand(H, E, 512)
        causal = torch.tensor([[s <= E - T + t for s in range(E)] for t in range(T)])
        ref_d = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=causal, scale=scale)
        torch.testing.assert_close(de[rows], ref_d.permute(1, 0, 2), rtol=1e-10, atol=1e-12)
        chosen = torch.zeros(T, E, dtype=torch.bool)
        for t in range(T):
            for s in idx[b * T + t].tolist():
                if s >= 0:
                    chosen[t, s] = True
        ref_s = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=chosen, scale=scale)
        torch.testing.assert_close(sp[rows], ref_s.permute(1, 0, 2), rtol=1e-10, atol=1e-12)
        logits = (Q @ K.transpose(-1, -2)) * scale
        ref_lse = torch.logsumexp(logits.masked_fill(~chosen, -math.inf), dim=-1).permute(1, 0)
        torch.testing.assert_close(lsp[rows], ref_lse, rtol=1e-12, atol=1e-12)


def test_sparse_mla_rejects_out_of_range_indices():
    q, kv, off = _mla_case(10, 1, 2)
    with pytest.raises(ValueError):
        oracle.sparse_mla(q, kv, off, torch.tensor([[10, -1]], dtype=torch.int32), 1, 1, 2, 2, 0.1)


# ---------------------------------------------------------------- cost model

def test_counted_macs_match_page_cost_model_and_break_even():
    """Per cached token the indexer costs 64*128 and MLA 128*576 multiply-adds;
    with top-2048 the sparse path breaks even with dense attention at n = 2304."""
    gold = json.load(open(os.path.join(GOLD, "cost_model.json")))
    assert gold["indexer_heads"] * gold["indexer_dim"] == gold["indexer_cost_per_token"]
    assert gold["mla_heads"] * gold["mla_dim"] == gold["mla_cost_per_token"]
    H, k = gold["mla_heads"], gold["topk"]

    def counted(n):
        inp = dsa_inputs.make_inputs(dsa_inputs.custom(end_pos=n, topk=k, H=H), "cpu")
        ci, cq, cd = oracle.Counter(), oracle.Counter(), oracle.Counter()
        sc = oracle.indexer_scores(inp.q_idx, inp.w, inp.k_idx, None, inp.offsets, 1, 1, n, macs=ci)
        idx = oracle.topk(sc, inp.offsets, 1, 1, k)
        oracle.sparse_mla(inp.q, inp.kv, inp.offsets, idx, 1, 1, H, k, 0.1, macs=cq)
        oracle.dense_mla(inp.q, inp.kv, inp.offsets, 1, 1, H, 0.1, macs=cd)
        # QK^T share of the attention counts (the page ignores the value product)
        qk_sparse = cq.value * 576 // (576 + 512)
        qk_dense = cd.value * 576 // (576 + 512)
        assert ci.value == n * gold["indexer_cost_per_token"]
        assert qk_sparse == min(n, k) * gold["mla_cost_per_token"]
        assert qk_dense == n * gold["mla_cost_per_token"]
        return ci.value + qk_sparse, qk_dense

    n0 = gold["break_even_n"]
    sparse, dense = counted(n0)
    assert sparse == dense
    s_lo, d_lo = counted(n0 - 64)
    s_hi, d_hi = counted(n0 + 64)
    assert s_lo > d_lo and s_hi < d_hi


# ---------------------------------------------------------------- whole path

def test_tiny_workload_end_to_end_invariants():
    inp = dsa_inputs.make_inputs(dsa_inputs.WORKLOADS["tiny"], "cpu")
    sc, idx, out, lse = oracle.decode_step(inp)
    assert sc.shape == (1, 256) and torch.isfinite(sc).all()
    sel = idx[0]
    assert (sel >= 0).sum().item() == 64
    assert torch.all(sel[1:] > sel[:-1])                       # ascending, distinct
    kept = set(sel.tolist())
    worst_kept = min(sc[0, s].item() for s in kept)
    assert all(sc[0, s].item() <= worst_kept for s in range(256) if s not in kept)
    assert out.shape == (1, 16, 512) and torch.isfinite(out).all()


# ---------------------------------------------------------------- act_quant (e4m3, block 128)
# The pages call act_quant(x, block_size, scale_fmt) without printing it
# ("Keep top-k positions", Indexer.forward).  Reading: scale = amax / 448 in
# fp32, code = nearest e4m3 value of x / scale, ties to the even code,
# saturating at +-448.  The pins below fix the encoder to the e4m3 value set
# (through the decoder, itself pinned against torch for every code above) and
# to hand-worked ties; the block quantiser to its closed forms.

def test_e4m3_encoder_inverts_the_decoder_for_every_finite_code():
    for code in range(256):
        if code & 0x7F == 0x7F:
            continue  # NaN
        assert oracle.e4m3_encode(oracle.e4m3_to_f64(code)) == code, hex(code)


@pytest.mark.parametrize("x,code", [
    (448.0, 0x7E), (1e6, 0x7E), (-1e6, 0xFE),     # saturation at the largest finite value
    (1.0625, 0x38),                                # midway 1.0 (0x38) .. 1.125 (0x39): even code
    (1.1875, 0x3A),                                # midway 1.125 (0x39) .. 1.25 (0x3A): even code
    (2.0 ** -10, 0x00),                            # midway 0 .. 2^-9 (smallest subnormal): even code
    (1.5 * 2.0 ** -10, 0x01),                      # nearer 2^-9 than 0
    (3.0 * 2.0 ** -10, 0x02),                      # midway 2^-9 (0x01) .. 2^-8 (0x02): even code
    (-0.0, 0x80), (0.0, 0x00), (240.0, 0x77),
])
def test_e4m3_encoder_hand_worked_values(x, code):
    assert oracle.e4m3_encode(x) == code


def test_e4m3_encoder_matches_torch_cast_on_random_values():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(20000, generator=g) * 30, torch.randn(5000, generator=g) * 1e-3,
                   (torch.randint(-3000, 3000, (5000,), generator=g).float() + 0.5) / 64])  # many exact ties
    mine = torch.tensor([oracle.e4m3_encode(float(v)) for v in x], dtype=torch.uint8)
    ref = x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(mine, ref)


def test_quantize_blocks_closed_forms():
    g = torch.Generator().manual_seed(8)
    x = (torch.randn(6, 128, generator=g) * torch.tensor([1e-3, 0.1, 1, 10, 300, 1e4])[:, None]).to(torch.bfloat16)
    x[2] = 0  # all-zero block
    codes, scales = oracle.quantize_blocks(x)
    xf = x.float()
    amax = xf.abs().amax(dim=1)
    for i in range(6):
        if amax[i] == 0:
            assert scales[i] == 1.0 and torch.all(codes[i] == 0)
            continue
        assert scales[i] == (amax[i] / 448.0)  # fp32 division
        j = int(xf[i].abs().argmax())
        assert codes[i, j] & 0x7F == 0x7E  # the largest magnitude lands on +-448
        deq = torch.tensor([oracle.e4m3_to_f64(int(c)) for c in codes[i]], dtype=torch.float64) * float(scales[i])
        # within half an e4m3 step (relative 2^-4) of the original, or the subnormal spacing
        err = (deq - xf[i].double()).abs()
        assert torch.all(err <= torch.maximum(xf[i].double().abs() * 2 ** -4, torch.tensor(2.0 ** -10) * float(scales[i])))


def test_quantize_blocks_agrees_with_the_input_generator():
    """The seeded input module quantises the e4m3 workload with torch ops; the
    oracle's own quantiser must give the same bytes."""
    g = torch.Generator().manual_seed(9)
    x = (torch.randn(64, 128, generator=g) * 2).to(torch.bfloat16)
    c1, s1 = oracle.quantize_blocks(x)
    c2, s2 = dsa_inputs.quantize_e4m3_blocks(x)
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


# ---------------------------------------------------------------- indexer pre-stage (RoPE + Hadamard)

def _rope_tables(n_pos, base=10000.0):
    """cos/sin of pos * theta_i, theta_i = base^(-i/32): a freqs_cis table of
    the usual form (the pages give no base; any table works for the pins)."""
    theta = base ** (-torch.arange(32, dtype=torch.float64) / 32)
    ang = torch.arange(n_pos, dtype=torch.float64)[:, None] * theta[None]
    return torch.cos(ang).float(), torch.sin(ang).float()


def _identity_tables(n_pos):
    return torch.ones(n_pos, 32), torch.zeros(n_pos, 32)


def test_rotate_activation_is_the_sylvester_hadamard_matrix():
    # the transform alone (identity rope) equals scipy's Hadamard matrix / sqrt(128)
    import scipy.linalg
    Hm = torch.tensor(scipy.linalg.hadamard(128), dtype=torch.float64) / math.sqrt(128)
    x = _bf16((5, 3, 128), seed=70)
    c, s = _identity_tables(4)
    pos = torch.tensor([0, 1, 2, 3, 0], dtype=torch.int32)
    y = oracle.rope_hadamard(x, pos, c, s, round_bf16=False)
    ref = x.double() @ Hm.T
    assert torch.allclose(y, ref, rtol=0, atol=1e-12)


def test_rotate_activation_is_an_involution_and_keeps_the_norm():
    x = _bf16((4, 2, 128), seed=71, scale=3.0)
    c, s = _identity_tables(1)
    pos = torch.zeros(4, dtype=torch.int32)
    y = oracle.rope_hadamard(x, pos, c, s, round_bf16=False)
    assert torch.allclose(y.norm(dim=-1), x.double().norm(dim=-1), rtol=1e-13)
    # H/sqrt(128) is symmetric and orthogonal: applying it twice gives x back
    import scipy.linalg
    Hm = torch.tensor(scipy.linalg.hadamard(128), dtype=torch.float64) / math.sqrt(128)
    assert torch.allclose(y @ Hm, x.double(), atol=1e-12)


@pytest.mark.parametrize("i", [0, 5, 31])
def test_rope_pairs_entry_i_with_entry_i_plus_32(i):
    # not interleaved: e_i -> cos at i, sin at i+32; e_{i+32} -> -sin at i, cos at i+32
    import scipy.linalg
    Hm = torch.tensor(scipy.linalg.hadamard(128), dtype=torch.float64) / math.sqrt(128)
    c, s = _rope_tables(8)
    p = 7
    x = torch.zeros(2, 1, 128)
    x[0, 0, i] = 1.0
    x[1, 0, i + 32] = 1.0
    y = oracle.rope_hadamard(x.to(torch.bfloat16), torch.tensor([p, p], dtype=torch.int32), c, s, round_bf16=False)
    u = y @ Hm  # undo the (symmetric, orthogonal) transform: the rope output
    want0 = torch.zeros(128, dtype=torch.float64)
    want0[i], want0[i + 32] = float(c[p, i]), float(s[p, i])
    want1 = torch.zeros(128, dtype=torch.float64)
    want1[i], want1[i + 32] = -float(s[p, i]), float(c[p, i])
    assert torch.allclose(u[0, 0], want0, atol=1e-12)
    assert torch.allclose(u[1, 0], want1, atol=1e-12)


def test_rope_leaves_the_second_half_alone_and_rotates_by_relative_position():
    import scipy.linalg
    Hm = torch.tensor(scipy.linalg.hadamard(128), dtype=torch.float64) / math.sqrt(128)
    c, s = _rope_tables(64)
    q = _bf16((1, 1, 128), seed=72)
    k = _bf16((1, 1, 128), seed=73)
    uq = oracle.rope_hadamard(q, torch.tensor([10], dtype=torch.int32), c, s, round_bf16=False) @ Hm
    assert torch.allclose(uq[0, 0, 64:], q[0, 0, 64:].double(), atol=0)  # the non-rope half passes through
    # <R_p q, R_p' k> depends only on p - p' (the table holds angles pos * theta)
    dots = []
    for p, pp in [(10, 3), (20, 13), (40, 33)]:
        yq = oracle.rope_hadamard(q, torch.tensor([p], dtype=torch.int32), c, s, round_bf16=False)
        yk = oracle.rope_hadamard(k, torch.tensor([pp], dtype=torch.int32), c, s, round_bf16=False)
        dots.append(float((yq * yk).sum()))
    assert max(dots) - min(dots) < 1e-5 * max(1.0, abs(dots[0]))


def test_rope_hadamard_bf16_rounding_points():
    # with rounding: every output is a bf16 value, within the error the two
    # rounding points allow of the exact result
    c, s = _rope_tables(32)
    x = _bf16((6, 4, 128), seed=74)
    pos = torch.tensor([0, 3, 7, 15, 31, 1], dtype=torch.int32)
    yr = oracle.rope_hadamard(x, pos, c, s, round_bf16=True)
    ye = oracle.rope_hadamard(x, pos, c, s, round_bf16=False)
    assert torch.equal(yr, yr.to(torch.bfloat16).double())
    rope_l1 = x[..., :64].double().abs().sum(-1, keepdim=True) * 1.42  # |a c - b s| + |a s + b c| <= 1.42 (|a| + |b|)
    bound = 2.0 ** -8 * ye.abs() + 2.0 ** -9 * rope_l1 / math.sqrt(128) + 1e-12
    assert bool(((yr - ye).abs() <= bound).all())
    assert bool(((yr - ye).abs() > 0).any())  # the rounding is really applied


def test_rope_hadamard_rejects_positions_outside_the_table():
    c, s = _rope_tables(4)
    x = _bf16((2, 1, 128), seed=75)
    with pytest.raises(ValueError):
        oracle.rope_hadamard(x, torch.tensor([0, 4], dtype=torch.int32), c, s)


def test_rope_hadamard_vectors_of_a_row_share_its_position():
    # V vectors per row (the 64 heads of a query row) all use pos[row]
    c, s = _rope_tables(16)
    x = _bf16((3, 5, 128), seed=76)
    pos = torch.tensor([2, 9, 15], dtype=torch.int32)
    y = oracle.rope_hadamard(x, pos, c, s, round_bf16=False)
    for r in range(3):
        for v in range(5):
            one = oracle.rope_hadamard(x[r:r + 1, v:v + 1].contiguous(), pos[r:r + 1], c, s, round_bf16=False)
            assert torch.equal(y[r, v], one[0, 0])
