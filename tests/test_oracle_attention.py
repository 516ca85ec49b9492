"""Pins of the attention oracle against things other than itself (CPU only).

* closed forms: a one-token context returns that token's V row exactly;
  constant keys (or a zero query) return the mean of V;
* a library routine: torch's scaled-dot-product attention in float64 on
  contiguous K/V (the paged result must equal contiguous attention);
* invariants: any physical placement of the pages gives the same bits;
  GQA equals MHA with each KV head repeated for its query heads;
* brute force: plain Python loops with math.exp on tiny inputs;
* the log-sum-exp merge of per-partition partials equals the unsplit result;
* planted mistakes (a copy of the oracle with one error each) fail these pins.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import c_oracle
from paged_kv_cache_320_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rand_bits(rng, shape, dtype):
    return synth.round_to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)


def make_paged(rng, lens, Hq, Hkv, d, bs, dtype, extra_blocks=3, canary=True):
    """Contiguous per-sequence K/V first, then scattered into a randomly placed pool.
    Returns (q, kc, vc, bt, lens, Kc, Vc) with Kc/Vc the contiguous originals."""
    nblk = [-(-n // bs) for n in lens]
    nb = sum(nblk) + extra_blocks
    mb = max(nblk) + 1
    perm = rng.permutation(nb)
    fill = synth.CANARY[dtype] if canary else 0
    kc = np.full((nb, Hkv, bs, d), fill, dtype=np.uint16)
    vc = np.full((nb, Hkv, bs, d), fill, dtype=np.uint16)
    bt = np.full((len(lens), mb), -1, dtype=np.int32)
    q = rand_bits(rng, (len(lens), Hq, d), dtype)
    Kc, Vc = [], []
    off = 0
    for s, n in enumerate(lens):
        K = rand_bits(rng, (n, Hkv, d), dtype)
        V = rand_bits(rng, (n, Hkv, d), dtype)
        Kc.append(K)
        Vc.append(V)
        bt[s, :nblk[s]] = perm[off:off + nblk[s]]
        off += nblk[s]
        for t in range(n):
            kc[bt[s, t // bs], :, t % bs, :] = K[t]
            vc[bt[s, t // bs], :, t % bs, :] = V[t]
    return q, kc, vc, bt, np.array(lens, dtype=np.int32), Kc, Vc


def sdpa_reference(q, Kc, Vc, dtype, scale, G):
    """torch scaled_dot_product_attention (float64) on the contiguous K/V."""
    outs = []
    for s in range(q.shape[0]):
        qs = torch.from_numpy(A.bits_to_f64(q[s], dtype))[:, None, :]          # [Hq,1,d]
        K = torch.from_numpy(A.bits_to_f64(Kc[s], dtype)).permute(1, 0, 2)      # [Hkv,n,d]
        V = torch.from_numpy(A.bits_to_f64(Vc[s], dtype)).permute(1, 0, 2)
        K = K.repeat_interleave(G, dim=0)
        V = V.repeat_interleave(G, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(qs, K, V, scale=scale)
        outs.append(o[:, 0, :].numpy())
    return np.stack(outs)


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
def test_one_token_context_returns_v_row(dtype):
    rng = np.random.default_rng(11)
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [1, 1, 1], 4, 2, 16, 4, dtype)
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 0.25, dtype)
    outc = c_oracle.paged_decode_attention(q, kc, vc, bt, lens, 0.25, dtype)
    for s in range(3):
        for h in range(4):
            expect = A.bits_to_f64(Vc[s][0, h // 2], dtype)
            np.testing.assert_array_equal(out[s, h], expect)
            np.testing.assert_array_equal(outc[s, h], expect)


def test_constant_keys_and_zero_query_give_mean_of_v():
    rng = np.random.default_rng(12)
    dtype = synth.BF16
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [5, 37], 2, 1, 8, 8, dtype)
    # constant keys: write one key row everywhere the sequences live
    key = rand_bits(rng, (8,), dtype)
    for s, n in enumerate(lens):
        for t in range(n):
            kc[bt[s, t // 8], 0, t % 8, :] = key
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 0.3, dtype)
    for s, n in enumerate(lens):
        mean = A.bits_to_f64(Vc[s][:, 0], dtype).mean(0)
        np.testing.assert_allclose(out[s, 0], mean, rtol=0, atol=1e-12)
    # zero query with random keys
    q0 = np.zeros_like(q)
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [9, 20], 2, 2, 8, 4, dtype)
    out = A.paged_decode_attention(q0, kc, vc, bt, lens, 1.0, dtype)
    outc = c_oracle.paged_decode_attention(q0, kc, vc, bt, lens, 1.0, dtype)
    for s in range(2):
        for h in range(2):
            mean = A.bits_to_f64(Vc[s][:, h], dtype).mean(0)
            np.testing.assert_allclose(out[s, h], mean, rtol=0, atol=1e-12)
            np.testing.assert_allclose(outc[s, h], mean, rtol=0, atol=1e-12)


def test_dominant_score_selects_its_value_row():
    rng = np.random.default_rng(13)
    dtype = synth.F16
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [30], 1, 1, 8, 16, dtype, canary=False)
    # q = e0 * 8; key 17 = e0 * 8, all others zero in dim 0 -> score gap 64*scale
    qv = np.zeros(8, np.float32); qv[0] = 8.0
    q[0, 0] = synth.round_to_bits(qv, dtype)
    for t in range(30):
        k = np.zeros(8, np.float32)
        if t == 17:
            k[0] = 8.0
        kc[bt[0, t // 16], 0, t % 16, :] = synth.round_to_bits(k, dtype)
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 1.0, dtype)
    np.testing.assert_allclose(out[0, 0], A.bits_to_f64(Vc[0][17, 0], dtype), atol=1e-20)


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
@pytest.mark.parametrize("Hq,Hkv,bs", [(4, 4, 16), (8, 2, 8), (8, 1, 32), (6, 3, 16)])
def test_equals_torch_sdpa_on_contiguous_kv(dtype, Hq, Hkv, bs):
    rng = np.random.default_rng(100 + Hq * 7 + Hkv + bs)
    lens = [1, bs - 1, bs, bs + 1, 3 * bs + 5, 70]
    d = 32
    q, kc, vc, bt, lens_a, Kc, Vc = make_paged(rng, lens, Hq, Hkv, d, bs, dtype)
    scale = 1.0 / math.sqrt(d)
    ref = sdpa_reference(q, Kc, Vc, dtype, scale, Hq // Hkv)
    out = A.paged_decode_attention(q, kc, vc, bt, lens_a, scale, dtype)
    outc = c_oracle.paged_decode_attention(q, kc, vc, bt, lens_a, scale, dtype)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(outc, ref, rtol=1e-12, atol=1e-12)


def test_placement_invariance_is_bit_exact():
    rng = np.random.default_rng(14)
    dtype = synth.BF16
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [3, 40, 17], 8, 2, 16, 8, dtype)
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 0.25, dtype)
    # move every physical page to a new place and rewrite the tables to match
    nb = kc.shape[0]
    new_pos = rng.permutation(nb)
    kc2 = np.empty_like(kc); vc2 = np.empty_like(vc)
    kc2[new_pos] = kc; vc2[new_pos] = vc
    bt2 = np.where(bt >= 0, new_pos[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = A.paged_decode_attention(q, kc2, vc2, bt2, lens, 0.25, dtype)
    np.testing.assert_array_equal(out, out2)
    outc = c_oracle.paged_decode_attention(q, kc, vc, bt, lens, 0.25, dtype)
    outc2 = c_oracle.paged_decode_attention(q, kc2, vc2, bt2, lens, 0.25, dtype)
    np.testing.assert_array_equal(outc, outc2)


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(15)
    dtype = synth.F16
    Hq, Hkv, G = 8, 2, 4
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [9, 33], Hq, Hkv, 16, 16, dtype)
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 0.25, dtype)
    kc_m = np.repeat(kc, G, axis=1)          # KV head h//G for query head h
    vc_m = np.repeat(vc, G, axis=1)
    out_m = A.paged_decode_attention(q, kc_m, vc_m, bt, lens, 0.25, dtype)
    np.testing.assert_array_equal(out, out_m)


def brute_force(q, kc, vc, bt, lens, scale, dtype):
    """Tiny-input brute force straight from the definition, pure Python loops."""
    B, Hq, d = q.shape
    Hkv, bs = kc.shape[1], kc.shape[2]
    G = Hq // Hkv
    f = lambda x: float(A.bits_to_f64(np.array([x], dtype=np.uint16), dtype)[0])
    out = [[[0.0] * d for _ in range(Hq)] for _ in range(B)]
    for s in range(B):
        n = int(lens[s])
        for h in range(Hq):
            hk = h // G
            scores = []
            for t in range(n):
                page, row = int(bt[s][t // bs]), t % bs
                scores.append(scale * sum(f(q[s, h, i]) * f(kc[page, hk, row, i]) for i in range(d)))
            mx = max(scores)
            w = [math.exp(x - mx) for x in scores]
            tot = sum(w)
            for i in range(d):
                acc = 0.0
                for t in range(n):
                    page, row = int(bt[s][t // bs]), t % bs
                    acc += w[t] * f(vc[page, hk, row, i])
                out[s][h][i] = acc / tot
    return np.array(out)


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
def test_brute_force_tiny(dtype):
    rng = np.random.default_rng(16)
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [1, 3, 5, 8], 4, 2, 4, 2, dtype)
    ref = brute_force(q, kc, vc, bt, lens, 0.7, dtype)
    np.testing.assert_allclose(A.paged_decode_attention(q, kc, vc, bt, lens, 0.7, dtype), ref,
                               rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(c_oracle.paged_decode_attention(q, kc, vc, bt, lens, 0.7, dtype),
                               ref, rtol=1e-12, atol=1e-13)


def test_log_sum_exp_merge_identity():
    rng = np.random.default_rng(17)
    qv = rng.standard_normal(16)
    K = rng.standard_normal((100, 16)) * 2
    V = rng.standard_normal((100, 16))
    full = A.softmax_attention(qv, K, V, 0.4)
    for part in (1, 7, 16, 64, 99, 100, 256):
        merged = A.merge_partitions(A.partition_partials(qv, K, V, 0.4, part))
        np.testing.assert_allclose(merged, full, rtol=1e-12, atol=1e-13)


def test_canary_outside_context_is_never_read():
    rng = np.random.default_rng(18)
    dtype = synth.BF16
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [5, 16, 17], 4, 4, 8, 16, dtype, canary=True)
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 0.3, dtype)
    outc = c_oracle.paged_decode_attention(q, kc, vc, bt, lens, 0.3, dtype)
    assert np.isfinite(out).all() and np.isfinite(outc).all()
    q2, kc2, vc2, bt2, lens2, _, _ = q, kc.copy(), vc.copy(), bt, lens, None, None
    kc2[kc2 == synth.CANARY[dtype]] = 0
    vc2[vc2 == synth.CANARY[dtype]] = 0
    np.testing.assert_array_equal(out, A.paged_decode_attention(q2, kc2, vc2, bt2, lens2, 0.3, dtype))


def test_zero_length_context_gives_zero():
    rng = np.random.default_rng(19)
    q, kc, vc, bt, lens, Kc, Vc = make_paged(rng, [4, 1], 2, 2, 8, 4, synth.F16)
    lens = np.array([0, 1], dtype=np.int32)
    out = A.paged_decode_attention(q, kc, vc, bt, lens, 0.3, synth.F16)
    outc = c_oracle.paged_decode_attention(q, kc, vc, bt, lens, 0.3, synth.F16)
    assert (out[0] == 0).all() and (outc[0] == 0).all()


# ----------------------------------------------------------------------------
# planted mistakes: each variant must fail the library-routine pin
# ----------------------------------------------------------------------------
def _variant(kind):
    def run(q, kc, vc, bt, lens, scale, dtype):
        B, Hq, d = q.shape
        Hkv, bs = kc.shape[1], kc.shape[2]
        G = Hq // Hkv
        out = np.zeros((B, Hq, d))
        for s in range(B):
            n = int(lens[s])
            t = np.arange(n)
            if kind == "page_row_swapped":
                pages, rows = bt[s][np.minimum(t % bs, bt.shape[1] - 1)], np.minimum(t // bs, bs - 1)
            else:
                pages, rows = bt[s][t // bs], t % bs
            for h in range(Hq):
                hk = (h % Hkv) if kind == "gqa_modulo" else h // G
                K = A.bits_to_f64(kc[pages, hk, rows], dtype)
                V = A.bits_to_f64(vc[pages, hk, rows], dtype)
                qv = A.bits_to_f64(q[s, h], dtype)
                if kind == "per_page_softmax":       # the page's literal loop
                    acc = np.zeros(d)
                    for a in range(0, n, bs):
                        x = K[a:a + bs] @ qv * scale
                        p = np.exp(x - x.max())
                        acc += (p / p.sum()) @ V[a:a + bs]
                    out[s, h] = acc
                    continue
                sc = 1.0 if kind == "no_scale" else scale
                x = sc * (K @ qv)
                p = np.exp(x - x.max())
                out[s, h] = p @ V / p.sum()
        return out
    return run


@pytest.mark.parametrize("kind", ["per_page_softmax", "no_scale", "gqa_modulo", "page_row_swapped"])
def test_planted_mistakes_fail_the_pins(kind):
    rng = np.random.default_rng(20)
    dtype = synth.BF16
    Hq, Hkv, bs, d = 8, 2, 4, 16
    lens = [3, 9, 14]
    q, kc, vc, bt, lens_a, Kc, Vc = make_paged(rng, lens, Hq, Hkv, d, bs, dtype, canary=False)
    scale = 1.0 / math.sqrt(d)
    ref = sdpa_reference(q, Kc, Vc, dtype, scale, Hq // Hkv)
    bad = _variant(kind)(q, kc, vc, bt, lens_a, scale, dtype)
    assert not np.allclose(bad, ref, rtol=1e-6, atol=1e-6)
    good = A.paged_decode_attention(q, kc, vc, bt, lens_a, scale, dtype)
    np.testing.assert_allclose(good, ref, rtol=1e-12, atol=1e-12)
