"""Pins of the oracle to things other than itself (library routines, closed forms,
invariants, brute force).  CPU only."""
import math

import pytest
import torch
import torch.nn.functional as F

import synth
from oracle import (OracleDecoder, argmax_lowest, attention_decode, e4m3_decode_table,
                    moe_route, rms_norm, rope_rotate, silu, swiglu_ffn)
from synth.configs import DecoderConfig

torch.manual_seed(0)


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_matches_library():
    x = torch.randn(5, 96)
    g = torch.rand(96) + 0.5
    ref = F.rms_norm(x, (96,), weight=g, eps=1e-5)
    assert torch.allclose(rms_norm(x, g, 1e-5), ref, rtol=1e-6, atol=1e-6)


def test_rmsnorm_closed_forms():
    # constant vector c: every entry becomes c / sqrt(c^2 + eps)
    for c in (0.25, -3.0):
        x = torch.full((64,), c)
        out = rms_norm(x, torch.ones(64), 1e-5)
        assert torch.allclose(out, torch.full((64,), c / math.sqrt(c * c + 1e-5)), rtol=1e-6)
    # unit gain gives unit RMS (eps negligible); scale invariance
    x = torch.randn(256) * 7
    y = rms_norm(x, torch.ones(256), 0.0)
    assert abs(float(y.pow(2).mean().sqrt()) - 1.0) < 1e-6
    assert torch.allclose(rms_norm(3.5 * x, torch.ones(256), 0.0), y, rtol=1e-5, atol=1e-6)


# --------------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    d, theta = 64, 1.0e4
    x = torch.randn(3, d)
    for pos in (0, 1, 17, 1000):
        z = torch.complex(x[:, : d // 2].double(), x[:, d // 2:].double())
        inv = theta ** (-2.0 * torch.arange(d // 2, dtype=torch.float64) / d)
        rot = z * torch.polar(torch.ones(d // 2, dtype=torch.float64), pos * inv)
        ref = torch.cat([rot.real, rot.imag], dim=-1).float()
        assert torch.allclose(rope_rotate(x, pos, theta), ref, rtol=1e-5, atol=1e-5)


def test_rope_invariants():
    d = 128
    q, k = torch.randn(d).double(), torch.randn(d).double()
    assert torch.equal(rope_rotate(q.float(), 0, 1e4), q.float())            # R(0) = I
    for m in (1, 50, 4097):
        assert abs(float(rope_rotate(q.float(), m, 1e4).norm()) - float(q.norm())) < 1e-4
    # relative position: <R(m) q, R(n) k> depends on m - n only
    a = torch.dot(rope_rotate(q.float(), 7, 1e4), rope_rotate(k.float(), 3, 1e4))
    b = torch.dot(rope_rotate(q.float(), 107, 1e4), rope_rotate(k.float(), 103, 1e4))
    assert abs(float(a - b)) < 1e-3


# ---------------------------------------------------------------- attention

def _sdpa_gqa(q, K, V):
    n_q, n_kv = q.shape[0], K.shape[0]
    Ke = K.float().repeat_interleave(n_q // n_kv, dim=0)
    Ve = V.float().repeat_interleave(n_q // n_kv, dim=0)
    out = F.scaled_dot_product_attention(q[:, None, :], Ke, Ve)      # [n_q][1][d]
    return out[:, 0]


@pytest.mark.parametrize("n_q,n_kv,T,d", [(4, 2, 129, 64), (32, 8, 300, 128), (8, 8, 5, 64)])
def test_attention_matches_library_sdpa(n_q, n_kv, T, d):
    q = torch.randn(n_q, d) * 2
    K = torch.randn(n_kv, T, d).to(torch.bfloat16)
    V = torch.randn(n_kv, T, d).to(torch.bfloat16)
    assert torch.allclose(attention_decode(q, K, V), _sdpa_gqa(q, K, V), rtol=1e-5, atol=1e-5)


def test_attention_special_cases():
    d = 64
    q = torch.randn(4, d)
    K = torch.randn(2, 1, d)
    V = torch.randn(2, 1, d)
    out = attention_decode(q, K, V)                                  # T = 1 -> output = v
    assert torch.allclose(out[0], V[0, 0]) and torch.allclose(out[3], V[1, 0])
    # one dominant score selects that V row; heads 0,1 read kv head 0, heads 2,3 kv head 1
    K = torch.zeros(2, 6, d)
    K[0, 4, 0] = 1.0
    K[1, 2, 0] = 1.0
    V = torch.randn(2, 6, d)
    q = torch.zeros(4, d)
    q[:, 0] = 1e4
    out = attention_decode(q, K, V)
    assert torch.allclose(out[1], V[0, 4], atol=1e-6)
    assert torch.allclose(out[2], V[1, 2], atol=1e-6)


def test_softmax_invariants_through_attention():
    # uniform scores -> mean of V rows; adding a constant to all scores changes nothing
    d = 64
    V = torch.randn(1, 10, d)
    out = attention_decode(torch.zeros(2, d), torch.randn(1, 10, d), V)
    assert torch.allclose(out[0], V[0].mean(0), atol=1e-6)
    q = torch.randn(1, d)
    K = torch.randn(1, 10, d)
    K2 = K + q / q.norm() ** 2 * 5.0 * math.sqrt(d)                  # shifts every score by 5
    assert torch.allclose(attention_decode(q, K, V), attention_decode(q, K2, V), atol=1e-4)


# ------------------------------------------------------------------- SwiGLU

def test_silu_matches_library_and_closed_forms():
    z = torch.linspace(-30, 30, 1001)
    assert torch.allclose(silu(z), F.silu(z), rtol=1e-6, atol=1e-7)
    assert float(silu(torch.tensor(0.0))) == 0.0
    assert abs(float(silu(torch.tensor(1.0))) - 0.7310585786300049) < 1e-7
    assert abs(float(silu(torch.tensor(40.0))) - 40.0) < 1e-5
    assert abs(float(silu(torch.tensor(-40.0)))) < 1e-12


def test_swiglu_structured():
    # diagonal gate/up and a permutation down projection: closed form per index
    n = 6
    a, b = torch.randn(n), torch.randn(n)
    sigma = [2, 0, 5, 1, 4, 3]
    wd = torch.zeros(n, n)
    for i, j in enumerate(sigma):
        wd[i, j] = 1.0
    xn = torch.randn(n)
    out = swiglu_ffn(xn, torch.diag(a), torch.diag(b), wd)
    for i, j in enumerate(sigma):
        z = float(a[j] * xn[j])
        assert abs(float(out[i]) - (z / (1 + math.exp(-z))) * float(b[j] * xn[j])) < 1e-5


# ---------------------------------------------------------------------- MoE

def test_moe_route_topk_vs_full_sort_and_ties():
    logits = torch.randn(64)
    ids, w, p = moe_route(logits, 8)
    assert abs(float(p.sum()) - 1.0) < 1e-6
    ref = torch.topk(torch.softmax(logits, 0), 8)
    assert ids == ref.indices.tolist()
    assert torch.allclose(torch.tensor(w), ref.values)
    # ties go to the lower expert id
    tied = torch.zeros(16)
    tied[[3, 9, 12]] = 2.0
    ids, _, _ = moe_route(tied, 2)
    assert ids == [3, 9]
    ids, _, _ = moe_route(torch.zeros(16), 4)
    assert ids == [0, 1, 2, 3]


def test_moe_single_expert_reduces_to_dense():
    base = DecoderConfig(name="t", n_layers=1, hidden=128, n_q_heads=2, n_kv_heads=1, head_dim=64,
                         ffn=256, vocab=300, kv_len=4, steps=2)
    moe = base.with_(ffn=0, n_experts=1, top_k=1, n_shared_experts=0, expert_ffn=256)
    wd = synth.make_weights(base)
    wm = synth.make_weights(moe)
    for k in ("w_gate", "w_up", "w_down"):
        wm[f"layers.0.experts.0.{k}"] = wd[f"layers.0.{k}"]
    dense, sparse = OracleDecoder(base, wd, 1), OracleDecoder(moe, wm, 1)
    for t in (5, 17, 299):
        ld, _ = dense.step([t])
        ls, _ = sparse.step([t])
        assert torch.allclose(ld, ls, rtol=1e-6, atol=1e-6)
        assert sparse.last_experts[0] == [[0]]


# ---------------------------------------------------------------------- FP8

def test_e4m3_table_matches_library_and_format():
    table = e4m3_decode_table()
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    nan = torch.isnan(lib)
    assert torch.equal(torch.isnan(table), nan)
    assert nan.sum() == 2 and bool(nan[0x7F]) and bool(nan[0xFF])
    assert torch.equal(table[~nan], lib[~nan])
    assert float(table[0x38]) == 1.0 and float(table[0x7E]) == 448.0
    assert float(table[0x01]) == 2.0 ** -9 and float(table[0xFE]) == -448.0
    assert float(table[0x80]) == 0.0


def test_fp8_quantisation_roundtrip_within_half_ulp():
    w = synth.normal_bf16(0, "q", (256, 384), 0.02)
    codes, scales = synth.quantize_fp8_blocks(w)
    deq = (e4m3_decode_table()[codes.long()].view(2, 128, 3, 128) * scales[:, None, :, None]).view(256, 384)
    rel = ((deq - w.float()).abs() / w.float().abs().clamp_min(1e-6))
    full_scale = scales.repeat_interleave(128, 0).repeat_interleave(128, 1)
    big = (w.float() / full_scale).abs() >= 2.0 ** -6                   # e4m3 normal range
    assert float(rel[big].max()) <= 2.0 ** -4 + 1e-6                   # 3 mantissa bits: half ulp
    assert float(codes.view(torch.float8_e4m3fn).float().abs().max()) == 448.0


# ------------------------------------------------------------------- argmax

def test_argmax_lowest_index_on_ties():
    v = torch.tensor([1.0, 3.0, 2.0, 3.0, 3.0])
    assert argmax_lowest(v) == 1
    v = torch.randn(1000)
    assert argmax_lowest(v) == int(torch.argmax(v))


# ------------------------------------------------------------ whole model

def _tiny(**kw):
    return synth.get_config("tiny", **kw)


def test_zero_layers_reduces_to_norm_and_lm_head():
    cfg = _tiny(n_layers=0)
    w = synth.make_weights(cfg, norm_std=0.1)
    m = OracleDecoder(cfg, w, 1)
    for t in (0, 7, 4095):
        logits, hidden = m.step([t])
        e = w["embed"][t].float()
        ref = F.linear(F.rms_norm(e, (cfg.hidden,), w["final_norm"], cfg.rms_eps), w["lm_head"].float())
        assert torch.allclose(hidden[0], e)
        assert torch.allclose(logits[0], ref, rtol=1e-5, atol=1e-6)


def test_structured_layer_closed_form():
    """One layer whose projections select / permute entries (every matrix non-square).

    Catches a transposed operand, a dropped residual, a wrong GQA group or a
    norm taken from the wrong vector: the expected output is built by index
    arithmetic only.
    """
    H, nq, nkv, d, Fw, V = 8, 2, 1, 2, 6, 16
    cfg = DecoderConfig(name="s", n_layers=1, hidden=H, n_q_heads=nq, n_kv_heads=nkv, head_dim=d,
                        ffn=Fw, vocab=V, kv_len=0, steps=3, rms_eps=1e-5)
    w = synth.make_weights(cfg)
    wq = torch.zeros(nq * d, H); wq[0, 0] = wq[1, 1] = wq[2, 2] = wq[3, 3] = 1.0
    wk = torch.zeros(nkv * d, H); wk[0, 4] = wk[1, 5] = 1.0
    wv = torch.zeros(nkv * d, H); wv[0, 6] = wv[1, 7] = 1.0
    wo = torch.zeros(H, nq * d)
    so = [3, 0, 2, 1, 0, 3, 1, 2]
    for i, j in enumerate(so):
        wo[i, j] = 1.0 if i < 4 else -1.0
    wg = torch.zeros(Fw, H); wu = torch.zeros(Fw, H); wdn = torch.zeros(H, Fw)
    sg, su = [1, 3, 5, 7, 0, 2], [2, 2, 4, 6, 1, 0]
    for f in range(Fw):
        wg[f, sg[f]] = 1.5
        wu[f, su[f]] = -0.5
    sd = [5, 4, 3, 2, 1, 0, 5, 4]
    for i, f in enumerate(sd):
        wdn[i, f] = 1.0
    lm = torch.zeros(V, H)
    for t in range(V):
        lm[t, t % H] = 1.0 if t < H else -2.0
    for name, t in (("wq", wq), ("wk", wk), ("wv", wv), ("wo", wo), ("w_gate", wg),
                    ("w_up", wu), ("w_down", wdn)):
        w[f"layers.0.{name}"] = t.to(torch.bfloat16)
    w["lm_head"] = lm.to(torch.bfloat16)
    m = OracleDecoder(cfg, w, 1, max_seq=4)

    def norm(v):
        r = 1.0 / math.sqrt(sum(a * a for a in v) / len(v) + 1e-5)
        return [a * r for a in v]

    def rot(p, pos):   # d = 2: one pair, theta_0 = 1
        c, s = math.cos(pos), math.sin(pos)
        return [p[0] * c - p[1] * s, p[0] * s + p[1] * c]

    ks, vs = [], []
    for pos, tok in enumerate([3, 11, 6]):
        x = [float(a) for a in w["embed"][tok].float()]
        xn = norm(x)
        q = [rot(xn[0:2], pos), rot(xn[2:4], pos)]
        ks.append([float(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)) for a in rot(xn[4:6], pos)])
        vs.append([float(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)) for a in xn[6:8]])
        o = []
        for h in range(nq):               # both q heads read kv head 0
            sc = [(q[h][0] * k[0] + q[h][1] * k[1]) / math.sqrt(d) for k in ks]
            mx = max(sc)
            e = [math.exp(s - mx) for s in sc]
            o += [sum(e[t] * vs[t][i] for t in range(len(e))) / sum(e) for i in range(d)]
        x1 = [x[i] + (o[so[i]] if i < 4 else -o[so[i]]) for i in range(H)]
        x1n = norm(x1)
        hmid = [(1.5 * x1n[sg[f]]) / (1 + math.exp(-1.5 * x1n[sg[f]])) * (-0.5 * x1n[su[f]])
                for f in range(Fw)]
        x2 = [x1[i] + hmid[sd[i]] for i in range(H)]
        x2n = norm(x2)
        ref = [x2n[t % H] * (1.0 if t < H else -2.0) for t in range(V)]
        logits, hidden = m.step([tok])
        assert torch.allclose(hidden[0], torch.tensor(x2), rtol=1e-5, atol=1e-5), pos
        assert torch.allclose(logits[0], torch.tensor(ref), rtol=1e-5, atol=1e-5), pos
        assert int(m.pos[0]) == pos + 1


def test_incremental_decode_equals_full_recompute():
    cfg = _tiny(n_layers=2)
    w = synth.make_weights(cfg, norm_std=0.1)
    toks = synth.make_prompt(cfg.with_(kv_len=12))                 # [1][13]
    full = OracleDecoder(cfg, w, 1, max_seq=16)
    ref = full.forward_sequence(toks)[0]                              # [13][V]
    inc = OracleDecoder(cfg, w, 1, max_seq=16)
    for t in range(toks.shape[1]):
        logits, _ = inc.step([int(toks[0, t])])
        assert torch.allclose(logits[0], ref[t], rtol=1e-4, atol=1e-5), t
    T = toks.shape[1]
    assert torch.equal(inc.K[:, :, :, :T], full.K[:, :, :, :T]) or \
        float((inc.K[:, :, :, :T].float() - full.K[:, :, :, :T].float()).abs().max()) < 2e-2
    assert torch.allclose(inc.V[:, :, :, :T].float(), full.V[:, :, :, :T].float(), atol=2e-2)


def test_gqa_with_equal_heads_is_mha():
    cfg = _tiny(n_layers=1, n_kv_heads=4)
    w = synth.make_weights(cfg)
    m = OracleDecoder(cfg, w, 1, max_seq=8)
    q = torch.randn(4, 64)
    K = torch.randn(4, 7, 64).to(torch.bfloat16)
    V = torch.randn(4, 7, 64).to(torch.bfloat16)
    ref = F.scaled_dot_product_attention(q[:, None], K.float(), V.float())[:, 0]
    assert torch.allclose(attention_decode(q, K, V), ref, atol=1e-5)
    logits, _ = m.step([1])
    assert logits.shape == (1, cfg.vocab)


def test_batch_sequences_are_independent():
    cfg = _tiny(n_layers=1, batch=2)
    w = synth.make_weights(cfg)
    mb = OracleDecoder(cfg, w, 2, max_seq=8)
    m0 = OracleDecoder(cfg, w, 1, max_seq=8)
    m1 = OracleDecoder(cfg, w, 1, max_seq=8)
    for a, b in ((3, 9), (100, 7)):
        lb, _ = mb.step([a, b])
        l0, _ = m0.step([a])
        l1, _ = m1.step([b])
        assert torch.equal(lb[0], l0[0]) and torch.equal(lb[1], l1[0])


# ------------------------------------------------- FP8 weights inside the model

def _bare_oracle(weights):
    """An oracle over a hand-made weight dict (only W() is exercised)."""
    cfg = DecoderConfig(name="w", n_layers=1, hidden=128, n_q_heads=2, n_kv_heads=1, head_dim=64,
                        ffn=128, vocab=8, kv_len=0, steps=1)
    return OracleDecoder(cfg, weights, 1, max_seq=1)


def test_oracle_fp8_dequant_by_index_on_a_2x3_block_grid():
    # 256 x 384 e4m3 codes: a 2 x 3 grid of 128x128 blocks, each with its own
    # scale; every element must be table[code] * scale[row // 128][col // 128]
    # (a transposed or mis-broadcast scale index fails on this non-square grid)
    N, K = 256, 384
    r = torch.arange(N)[:, None]
    c = torch.arange(K)[None, :]
    codes = ((r * 7 + c * 13) % 126).to(torch.uint8)          # finite codes only (0x7F is NaN)
    codes[200, 300] = 0xFE                                     # -448
    codes[5, 129] = 0x80                                       # -0
    scales = torch.tensor([[0.5, 1.5, 3.0], [0.25, 2.0, 5.0]], dtype=torch.float32)
    o = _bare_oracle({"m": codes, "m.scale": scales})
    W = o.W("m")
    assert W.shape == (N, K) and W.dtype == torch.float32
    table = e4m3_decode_table()
    for (i, j) in [(0, 0), (127, 127), (128, 0), (0, 128), (127, 255), (128, 256), (255, 383), (200, 300),
                   (5, 129), (131, 17), (64, 200), (250, 130)]:
        want = float(torch.tensor(float(table[int(codes[i, j])]) * float(scales[i // 128, j // 128]),
                                  dtype=torch.float32))
        assert float(W[i, j]) == want, (i, j)
    # every block as a whole: block (bi, bj) / its scale is the decoded codes
    for bi in range(2):
        for bj in range(3):
            blk = W[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128] / scales[bi, bj]
            assert torch.equal(blk, table[codes[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128].long()])


def test_oracle_fp8_weights_reproduce_the_bf16_originals():
    # quantise seeded bf16 weights with the harness codec, widen them through the
    # oracle's W(): each element is the original within e4m3's half-ulp of its block
    w = synth.normal_bf16(0, "pin.fp8", (256, 384), 0.02)
    codes, scales = synth.quantize_fp8_blocks(w)
    W = _bare_oracle({"m": codes, "m.scale": scales}).W("m")
    full_scale = scales.repeat_interleave(128, 0).repeat_interleave(128, 1)
    q = w.float() / full_scale                                   # value in code units
    err = (W - w.float()).abs() / full_scale                     # error in code units
    normal = q.abs() >= 2.0 ** -6
    # normal range: 3 mantissa bits -> |err| <= 2^-4 relative; subnormals: spacing 2^-9
    assert bool((err[normal] <= q.abs()[normal] * 2.0 ** -4 * (1 + 1e-6)).all())
    assert bool((err[~normal] <= 2.0 ** -10 * (1 + 1e-6)).all())
    # and the block maximum is represented exactly (scale = amax / 448)
    amax = w.float().view(2, 128, 3, 128).abs().amax(dim=(1, 3))
    assert torch.allclose(W.view(2, 128, 3, 128).abs().amax(dim=(1, 3)), amax, rtol=1e-6)


# ----------------------------------------------------- MoE composition, k > 1

def _moe_structured():
    """A one-layer MoE whose router and experts select entries by index.

    H = 8, 4 routed experts (top-2) + 1 shared, expert width 4.  Router row e picks
    xn[e] times c_e; expert e's gate row f picks xn[(f + e) % H] times a_e, its up
    row f picks xn[(f + 2e + 1) % H] times b_e, and its down projection sends
    h[(i + e) % 4] to output i.  The shared expert is built the same way with e = 4.
    """
    H, E, Fe = 8, 4, 4
    cfg = DecoderConfig(name="m", n_layers=1, hidden=H, n_q_heads=2, n_kv_heads=1, head_dim=4, ffn=0,
                        vocab=16, kv_len=0, steps=1, n_experts=E, top_k=2, n_shared_experts=1, expert_ffn=Fe)
    w = synth.make_weights(cfg)
    c = [1.0, 3.0, -2.0, 0.5]
    a = [1.5, -0.75, 1.25, 2.0, 0.5]
    bb = [-0.5, 1.0, 0.25, -1.5, 1.75]
    router = torch.zeros(E, H)
    for e in range(E):
        router[e, e] = c[e]
    w["layers.0.router"] = router.to(torch.bfloat16)

    def expert(e):
        g, u, d = torch.zeros(Fe, H), torch.zeros(Fe, H), torch.zeros(H, Fe)
        for f in range(Fe):
            g[f, (f + e) % H] = a[e]
            u[f, (f + 2 * e + 1) % H] = bb[e]
        for i in range(H):
            d[i, (i + e) % Fe] = 1.0
        return g, u, d

    for e in range(E + 1):
        g, u, d = expert(e)
        q = f"layers.0.experts.{e}." if e < E else "layers.0.shared.0."
        w[q + "w_gate"], w[q + "w_up"], w[q + "w_down"] = (t.to(torch.bfloat16) for t in (g, u, d))
    return cfg, w, c, a, bb


def test_moe_topk2_plus_shared_expert_closed_form():
    cfg, w, c, a, bb = _moe_structured()
    H, E, Fe = cfg.hidden, cfg.n_experts, cfg.expert_ffn
    o = OracleDecoder(cfg, w, 1, max_seq=2)
    for xn_vals in ([0.3, 0.9, -0.4, 1.1, -0.2, 0.7, 0.05, -1.3], [2.0, -0.1, 0.6, 0.2, 1.0, -0.8, 0.4, 0.9]):
        xn = torch.tensor(xn_vals, dtype=torch.float32)
        # hand routing: logits z_e = c_e xn[e], softmax, top-2 by probability (lower id on ties)
        z = [c[e] * xn_vals[e] for e in range(E)]
        mz = max(z)
        ez = [math.exp(v - mz) for v in z]
        p = [v / sum(ez) for v in ez]
        top = sorted(range(E), key=lambda e: (-p[e], e))[:2]

        def h(e):
            out = []
            for f in range(Fe):
                g = a[e] * xn_vals[(f + e) % H]
                out.append(g / (1 + math.exp(-g)) * bb[e] * xn_vals[(f + 2 * e + 1) % H])
            return out

        want = [sum(p[e] * h(e)[(i + e) % Fe] for e in top) + h(E)[(i + E) % Fe] for i in range(H)]
        o._router_probs = []
        got, ids = o._ffn(0, xn)
        assert ids == top
        assert torch.allclose(got, torch.tensor(want, dtype=torch.float32), rtol=1e-5, atol=1e-6), (got, want)
        assert torch.allclose(o._router_probs[0], torch.tensor(p, dtype=torch.float32), rtol=1e-6)


def test_moe_incremental_decode_equals_full_recompute():
    cfg = DecoderConfig(name="m", n_layers=2, hidden=128, n_q_heads=2, n_kv_heads=1, head_dim=64, ffn=0,
                        vocab=300, kv_len=9, steps=1, n_experts=4, top_k=2, n_shared_experts=1, expert_ffn=64)
    w = synth.make_weights(cfg, norm_std=0.1)
    toks = synth.make_prompt(cfg)                                   # [1][10]
    full = OracleDecoder(cfg, w, 1, max_seq=12)
    ref = full.forward_sequence(toks)[0]
    inc = OracleDecoder(cfg, w, 1, max_seq=12)
    for t in range(toks.shape[1]):
        logits, _ = inc.step([int(toks[0, t])])
        assert torch.allclose(logits[0], ref[t], rtol=1e-4, atol=1e-5), t
    T = toks.shape[1]
    assert torch.allclose(inc.K[:, :, :, :T].float(), full.K[:, :, :, :T].float(), atol=2e-2)
    assert torch.allclose(inc.V[:, :, :, :T].float(), full.V[:, :, :, :T].float(), atol=2e-2)


# ----------------------------------------------------------- e4m3 encoding

def test_e4m3_encoder_matches_library_rounding():
    # the oracle's encoder (written from the format) against the library's
    # conversion of the same values clamped to the finite range (satfinite)
    from oracle import e4m3_encode
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 300.0)]
                  + [torch.tensor([0.0, -0.0, 448.0, -448.0, 449.0, 1e6, -1e6, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11])])
    lib = x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(e4m3_encode(x), lib)


def test_e4m3_encoder_ties_go_to_the_even_code():
    from oracle import e4m3_decode_table, e4m3_encode
    t = e4m3_decode_table()
    for c in (0x01, 0x08, 0x10, 0x30, 0x38, 0x3B, 0x50, 0x70, 0x7C):
        mid = float((t[c] + t[c + 1]) / 2)                  # halfway between codes c and c + 1
        want = c if c % 2 == 0 else c + 1
        assert int(e4m3_encode(torch.tensor([mid]))) == want, hex(c)
        assert int(e4m3_encode(torch.tensor([-mid]))) == want | 0x80, hex(c)


def test_fp8_kv_round_is_code_times_a_power_of_two():
    from oracle.decoder import kv_round
    from oracle import e4m3_decode_table
    table = e4m3_decode_table()
    finite = table[~torch.isnan(table)]
    x = torch.randn(4, 128) * 0.4
    for scale in (2.0 ** -7, 2.0 ** -3):
        r = kv_round(x, "fp8_e4m3", scale).float()
        q = r / scale
        assert bool(torch.isin(q, finite).all())          # every entry is an e4m3 value times the scale
        assert torch.equal(kv_round(r, "fp8_e4m3", scale).float(), r)   # idempotent
        # nearest: no e4m3 value is closer to x / scale than the chosen one
        d = (x / scale).clamp(-448, 448)
        err = (q - d).abs()
        best = (finite[None, None, :] - d[..., None]).abs().min(dim=-1).values
        assert bool((err <= best + 1e-7).all())
    with pytest.raises(AssertionError):
        kv_round(x, "fp8_e4m3", 0.3)                     # not a power of two


# ----------------------------------------------------------- NVFP4 weights

def test_e2m1_table_is_the_published_value_set():
    # OCP MX v1.0 lists the FP4 (E2M1) magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for
    # codes 0..7; codes 8..15 are their negatives (sign bit 3)
    from oracle import e2m1_decode_table
    t = e2m1_decode_table()
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert t[:8].tolist() == mags
    assert t[8:].tolist() == [-m for m in mags]
    assert bool(torch.signbit(t[8]))


def test_nvfp4_dequant_by_index():
    # distinct codes and block scales on a 3 x 64 matrix (4 blocks per row): each
    # element is the nibble of its byte (even element low) x its row's block scale
    # x the tensor scale
    from oracle import e2m1_decode_table, e4m3_decode_table, nvfp4_dequant
    g = torch.Generator().manual_seed(11)
    N, K = 3, 64
    codes = torch.randint(0, 256, (N, K // 2), generator=g).to(torch.uint8)
    scale_codes = torch.tensor([[0x30, 0x38, 0x40, 0x29], [0x31, 0x3F, 0x08, 0x50], [0x00, 0x44, 0x36, 0x3A]],
                               dtype=torch.uint8)
    gs = 0.375
    got = nvfp4_dequant(codes, scale_codes, gs)
    e2 = e2m1_decode_table().tolist()
    e4 = e4m3_decode_table().tolist()
    for r in range(N):
        for k in range(K):
            byte = int(codes[r, k // 2])
            nib = byte & 0xF if k % 2 == 0 else byte >> 4
            want = e2[nib] * e4[int(scale_codes[r, k // 16])] * gs
            assert float(got[r, k]) == want, (r, k)


def test_nvfp4_quantisation_picks_the_nearest_code():
    # the synthetic quantiser (input preparation) against brute force: every
    # element's value is, among the 16 codes times its block's scale, one nearest
    # to the weight; the oracle's dequantisation of its output stays within half
    # the largest code spacing (1 x scale) of the weight, below the saturation bound
    import synth
    from oracle import e4m3_decode_table, nvfp4_dequant
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(8, 256, generator=g) * 0.02).to(torch.bfloat16)
    w[0, :16] = 0                                          # an all-zero block
    codes, sc, gs = synth.quantize_nvfp4(w)
    deq = nvfp4_dequant(codes, sc, float(gs[0]))
    s = e4m3_decode_table()[sc.long()].repeat_interleave(16, dim=1) * float(gs[0])
    cand = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    wf = w.float()
    assert bool((deq[0, :16] == 0).all())
    for r in range(8):
        for k in range(256):
            if float(s[r, k]) == 0:
                continue
            opts = (torch.cat([cand, -cand]) * s[r, k] - wf[r, k]).abs()
            assert abs(float(deq[r, k]) - float(wf[r, k])) <= float(opts.min()) + 1e-6 * abs(float(wf[r, k])) + 1e-9, (r, k)
    # the block maximum maps to (about) 6: block scales are max|block| / 6 rounded to e4m3
    assert float((deq - wf).abs().max()) <= float(s.max()) * 1.0


def test_oracle_W_reads_nvfp4_weights():
    # OracleDecoder.W dispatches on the tensor-scale companion and returns the
    # dequantised matrix
    import synth
    from oracle import OracleDecoder, nvfp4_dequant
    cfg = synth.get_config("tiny", n_layers=1, weight_dtype="nvfp4")
    w = synth.make_weights(cfg)
    o = OracleDecoder(cfg, w, cfg.batch, max_seq=cfg.max_seq)
    name = "layers.0.wq"
    assert w[name].dtype == torch.uint8 and w[name].shape == (cfg.q_dim, cfg.hidden // 2)
    ref = nvfp4_dequant(w[name], w[name + ".scale"], float(w[name + ".gscale"][0]))
    assert torch.equal(o.W(name), ref)
    # and close to the bf16 weights it quantises (4-bit codes: ~10 % per element)
    wb = synth.normal_bf16(cfg.seed, name, (cfg.q_dim, cfg.hidden), cfg.init_std, "cpu").float()
    assert float((o.W(name) - wb).norm() / wb.norm()) < 0.15
