"""GPU parity of the KIVI-style low-bit cache against the CPU oracle
("KV Cache compression", 2.1 and 3.1 KIVI: K quantized per channel over groups
of positions, V per token, asymmetric 2-bit codes, the newest tokens kept in
full precision; "KV cache quantization: what FP8/INT8 K and V really give",
"Formats you will actually meet": the 4-bit variants).

Each sequence's complete 128-token groups go through kvq_kivi_append (one call
for all sequences), its residual tokens through kvq_append into a BF16 cache of
their own. Checked: the codes (unpacked from the documented page layout) and
the BF16 (s, z) pairs bit-exact against oracle/kivi.py, and the attention
output of kvq_kivi_decode_attn within max 4e-3 / mean 5e-4 of the oracle's FP64
attention over the dequantized groups followed by the BF16 residual.
"""

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import workloads as W
from oracle import attention as OA
from oracle import formats as OF
from oracle import kivi as OK

MAX_ABS, MEAN_ABS = 4e-3, 5e-4


def unpack_unit(words, bits):
    """16 codes of one packed unit (the header's bit order)."""
    out = np.zeros(16, dtype=np.uint8)
    for e in range(16):
        m, j = e >> 2, e & 3
        if bits == 2:
            out[e] = (int(words[0]) >> (8 * j + 2 * m)) & 3
        else:
            out[e] = (int(words[m >> 1]) >> (8 * j + 4 * (m & 1))) & 15
    return out


def unpack_k_page(page, D, bits):
    """[16 tokens][D] codes of one packed K page (uint8 bytes)."""
    w = page.view(np.uint32).reshape(-1, bits // 2)
    codes = np.zeros((16, D), dtype=np.uint8)
    for t in range(16):
        for c in range(D // 16):
            u = ((t >> 3) * (D // 16) + c) * 8 + (t & 7)
            codes[t, 16 * c:16 * c + 16] = unpack_unit(w[u], bits)
    return codes


def unpack_v_page(page, D, bits):
    w = page.view(np.uint32).reshape(-1, bits // 2)
    codes = np.zeros((16, D), dtype=np.uint8)
    for d in range(D):
        codes[:, d] = unpack_unit(w[d], bits)
    return codes


def _build(fmt, lens, Hk=2, G=4, D=128, seed=0, kv_mean=0.0, quantized=None):
    bits = kvq.KIVI_BITS[fmt]
    w = W.Workload("kivi", "fp8", batch=len(lens), n_q_heads=Hk * G, n_kv_heads=Hk, head_dim=D,
                   lengths="list", ctx=tuple(lens), kv_mean=kv_mean)
    rng = np.random.default_rng(seed)
    # quantized[b]: the sequence's tokens in complete groups (default: all of
    # its complete groups); the rest stays in the BF16 residual cache
    groups = [n // 128 for n in lens] if quantized is None else [m // 128 for m in quantized]
    res = [n - 128 * g for n, g in zip(lens, groups)]
    # low-bit pool: 8 blocks per group, shuffled; residual pool: its own blocks
    nq = max(1, sum(groups) * 8)
    perm = rng.permutation(nq)
    Wq = max(1, max(groups) * 8)
    qt = np.full((len(lens), Wq), -1, dtype=np.int32)
    at = 0
    for b, g in enumerate(groups):
        qt[b, :8 * g] = perm[at:at + 8 * g]
        at += 8 * g
    nr = max(1, sum((r + 15) // 16 for r in res))
    rperm = rng.permutation(nr)
    Wr = max(1, max((r + 15) // 16 for r in res))
    rt = np.full((len(lens), Wr), -1, dtype=np.int32)
    at = 0
    for b, r in enumerate(res):
        n = (r + 15) // 16
        rt[b, :n] = rperm[at:at + n]
        at += n
    d = kvq.dims(nq, Hk, Hk * G, D, Wq)
    rd = kvq.dims(nr, Hk, Hk * G, D, Wr)
    cache = kvq.KiviCache.allocate(fmt, d, rd)
    hist = [W.kv_history(w, b, seed) for b in range(w.batch)]
    Kq, Vq, Sq, Kr, Vr, Sr = [], [], [], [], [], []
    for b in range(w.batch):
        k, v = hist[b]
        m = groups[b] * 128
        pos = np.arange(m)
        Kq.append(k[:m]); Vq.append(v[:m])
        Sq.append(qt[b][pos // 16].astype(np.int64) * 16 + pos % 16)
        pos = np.arange(res[b])
        Kr.append(k[m:]); Vr.append(v[m:])
        Sr.append(rt[b][pos // 16].astype(np.int64) * 16 + pos % 16)
    if sum(groups):
        cache.append_groups(torch.cat(Kq).cuda(), torch.cat(Vq).cuda(),
                            torch.from_numpy(np.concatenate(Sq)).cuda())
    if sum(res):
        cache.residual.append(torch.cat(Kr).cuda(), torch.cat(Vr).cuda(),
                              torch.from_numpy(np.concatenate(Sr)).cuda())
    torch.cuda.synchronize()
    return w, bits, cache, qt, rt, hist, groups, res


def _check_codes(cache, bits, qt, hist, groups, b, D, Hk):
    k, v = hist[b]
    st = OK.quantize_sequence(k.float().numpy(), v.float().numpy(), bits=bits)
    kc = cache.k.cpu().numpy()
    vc = cache.v.cpu().numpy()
    km = cache.k_meta.float().cpu().numpy()
    vm = cache.v_meta.float().cpu().numpy()
    cpp = D // 8
    for g in range(groups[b]):
        for i in range(8):
            blk = qt[b][8 * g + i]
            for h in range(Hk):
                gk = unpack_k_page(kc[blk, h], D, bits)
                gv = unpack_v_page(vc[blk, h], D, bits)
                toks = slice(16 * i, 16 * i + 16)
                assert np.array_equal(gk, st["k_codes"][g, toks, h, :]), (b, g, i, h, "k codes")
                assert np.array_equal(gv, st["v_codes"][128 * g + 16 * i:128 * g + 16 * i + 16, h, :]), \
                    (b, g, i, h, "v codes")
                ch = slice(i * cpp, i * cpp + cpp)
                assert np.array_equal(OF.bf16_bits(km[blk, h, :cpp, 0]), OF.bf16_bits(st["k_s"][g, h, ch]))
                assert np.array_equal(OF.bf16_bits(km[blk, h, :cpp, 1]), OF.bf16_bits(st["k_z"][g, h, ch]))
                pos = slice(128 * g + 16 * i, 128 * g + 16 * i + 16)
                assert np.array_equal(OF.bf16_bits(vm[blk, h, :, 0]), OF.bf16_bits(st["v_s"][pos, h]))
                assert np.array_equal(OF.bf16_bits(vm[blk, h, :, 1]), OF.bf16_bits(st["v_z"][pos, h]))
    return st


def _run(fmt, lens, Hk=2, G=4, D=128, seed=0, kv_mean=0.0, check_codes=True, quantized=None):
    w, bits, cache, qt, rt, hist, groups, res = _build(fmt, lens, Hk, G, D, seed, kv_mean, quantized)
    g = torch.Generator().manual_seed(50 + seed)
    q = torch.randn(w.batch, Hk * G, D, generator=g).to(torch.bfloat16)
    ql = np.array([x * 128 for x in groups], dtype=np.int32)
    rl = np.array(res, dtype=np.int32)
    out = cache.decode(q.cuda(), torch.from_numpy(qt).cuda(), torch.from_numpy(ql).cuda(),
                       max(128, int(ql.max())) if ql.max() > 0 else 0,
                       torch.from_numpy(rt).cuda(), torch.from_numpy(rl).cuda(), int(rl.max()),
                       sm_scale=w.sm_scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.device_error() == 0
    errs = []
    for b in range(w.batch):
        k, v = hist[b]
        m = groups[b] * 128
        if quantized is None:
            st = (_check_codes(cache, bits, qt, hist, groups, b, D, Hk) if check_codes else
                  OK.quantize_sequence(k.float().numpy(), v.float().numpy(), bits=bits))
            K, V = OK.dequantize_sequence(st)
        else:
            # the first m tokens as groups, every later one in BF16
            st = OK.quantize_sequence(k[:m].float().numpy(), v[:m].float().numpy(), bits=bits)
            K, V = OK.dequantize_sequence(st)
            K = np.concatenate([K, k[m:].float().numpy().astype(np.float64)])
            V = np.concatenate([V, v[m:].float().numpy().astype(np.float64)])
        ref = OA.decode_attention(q[b:b + 1].float().numpy(), [(K, V)], w.sm_scale, Hk)[0]
        errs.append(np.abs(out[b].cpu().numpy().astype(np.float64) - ref).ravel())
    e = np.concatenate(errs)
    return float(e.max()), float(e.mean())


pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["kivi2", "kivi4"])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_kivi_parity(fmt, G):
    mx, mean = _run(fmt, [300, 128, 1000, 77, 2048, 256], G=G)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("fmt", ["kivi2", "kivi4"])
def test_kivi_head_dim_64_nonzero_mean(fmt):
    mx, mean = _run(fmt, [129, 640, 5], Hk=2, G=2, D=64, kv_mean=0.3)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


def test_kivi_long_contexts():
    """Several CTAs per sequence (split-K) and many groups."""
    mx, mean = _run("kivi2", [8192 + 50, 4096, 12000], G=8, check_codes=False)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("fmt", ["kivi2", "kivi4"])
def test_kivi_residual_longer_than_a_group(fmt):
    """Residuals of several hundred BF16 tokens (a caller that has not yet
    quantized complete groups): the residual attention runs over several
    128-token chunks, its online softmax moving between them; sequences with
    no quantized group at all and with no residual are mixed in."""
    lens = [900, 300, 2048, 129, 640]
    quantized = [256, 0, 2048, 0, 128]
    mx, mean = _run(fmt, lens, G=8, quantized=quantized)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
