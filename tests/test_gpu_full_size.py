"""Full-size workloads on the B200, in the launch configurations bench.py times, with
sampled outputs checked against the float64 oracle (the oracle recomputes the sampled
kv heads / queries completely, from the same inputs)."""
import math

import numpy as np
import pytest

import oracle
import workloads as W
import layout
import parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import kv_cache_vector_08_b200 as tq  # noqa: E402

DEV = torch.device("cuda", 0)


def _gen_kv(w, T, seed, B=None):
    """Device-side K/V [B, Hkv, T, D] bf16 with the workload's value distribution."""
    B = w.batch if B is None else B
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    shape = (B, w.kv_heads, T, w.head_dim)
    k = torch.randn(shape, generator=g, device=DEV)
    v = torch.randn(shape, generator=g, device=DEV)
    if w.outliers:
        for x, stream in ((k, W.STREAM_KEY_OUTLIERS), (v, W.STREAM_VALUE_OUTLIERS)):
            ch = W.outlier_channels(w.kv_heads, w.head_dim, w.outliers, seed, stream)
            for h in range(w.kv_heads):
                x[:, h, :, torch.tensor(ch[h], device=DEV)] *= w.outlier_factor
    if w.lognormal_sigma:
        k *= torch.exp(torch.randn((B, 1, T, 1), generator=g, device=DEV) * w.lognormal_sigma)
        v *= torch.exp(torch.randn((B, 1, T, 1), generator=g, device=DEV) * w.lognormal_sigma)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


class Cache:
    def __init__(self, w, B, max_len):
        self.w, self.B, self.max_len = w, B, max_len
        cap = B * w.kv_heads * max_len
        self.kctx, self.vctx, self.kc, self.vc, self.off = [], [], [], [], []
        for gi, (off, wd, kb, vb) in enumerate(w.groups):
            kx = tq.Context(wd, kb, 1000 + 2 * gi, tq.MODE_PROD)
            vx = tq.Context(wd, vb, 1001 + 2 * gi, tq.MODE_MSE)
            self.kctx.append(kx); self.vctx.append(vx)
            self.kc.append(tq.alloc_packed(kx, cap)); self.vc.append(tq.alloc_packed(vx, cap))
            self.off.append(off)
        self.off.append(w.head_dim)
        self.kp = [oracle.make_params(wd, kb, 1000 + 2 * gi, 0) for gi, (_, wd, kb, _) in enumerate(w.groups)]
        self.vp = [oracle.make_params(wd, vb, 1001 + 2 * gi, 1) for gi, (_, wd, _, vb) in enumerate(w.groups)]

    def write(self, K, V, t0, slots=None):
        """Quantize rows of K/V [B, Hkv, T', D] into token positions t0 .. t0+T'-1."""
        B, Hkv, Tn, D = K.shape
        Kf, Vf = K.reshape(-1, D), V.reshape(-1, D)
        if slots is None:
            b = torch.arange(B, device=DEV).view(B, 1, 1)
            h = torch.arange(Hkv, device=DEV).view(1, Hkv, 1)
            t = torch.arange(Tn, device=DEV).view(1, 1, Tn) + t0
            slots = ((b * Hkv + h) * self.max_len + t).reshape(-1).to(torch.int64)
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            tq.quantize_kv(self.kctx[gi], Kf[:, off:off + wd], self.kc[gi], slots=slots)
            tq.quantize_kv(self.vctx[gi], Vf[:, off:off + wd], self.vc[gi], slots=slots)

    def decode(self, q, seq_lens):
        sl = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
        return tq.decode_attention(self.kctx, self.vctx, self.off, q, self.kc, self.vc, sl, self.w.kv_heads,
                                   self.max_len, 1.0 / math.sqrt(self.w.head_dim))

    def check_head(self, K, V, q, out, b, hk, T, label):
        """Oracle over the full context of (b, hk): codes of every row, then the 4 heads'
        attention outputs (computed from the oracle's own quantization, with exempt rows
        reconciled to the GPU's indices)."""
        Hkv, rep, D = self.w.kv_heads, self.w.q_heads // self.w.kv_heads, self.w.head_dim
        slot0 = (b * Hkv + hk) * self.max_len
        rows = torch.arange(slot0, slot0 + T, device=DEV)
        kx = K[b, hk, :T].float().cpu().numpy().astype(np.float64)
        vx = V[b, hk, :T].float().cpu().numpy().astype(np.float64)
        kcodes, vcodes = [], []
        for gi, (off, wd, kb, vb) in enumerate(self.w.groups):
            c = self.kc[gi].codes[rows].cpu().numpy()
            parity.check_codes(self.kp[gi], kx[:, off:off + wd], c, self.kc[gi].norm[rows].float().cpu().numpy(),
                               self.kc[gi].rnorm[rows].float().cpu().numpy(), label + " keys g%d" % gi)
            ko = parity.reconciled_oracle_codes(self.kp[gi], kx[:, off:off + wd], c)
            kcodes.append({k: (None if ko[k] is None else ko[k][None, None]) for k in ("idx", "signs", "norm", "rnorm")})
            cv = self.vc[gi].codes[rows].cpu().numpy()
            parity.check_codes(self.vp[gi], vx[:, off:off + wd], cv, self.vc[gi].norm[rows].float().cpu().numpy(),
                               None, label + " values g%d" % gi)
            vo = parity.reconciled_oracle_codes(self.vp[gi], vx[:, off:off + wd], cv)
            vcodes.append({k: vo[k][None, None] for k in ("idx", "norm")})
        qn = q[b, hk * rep:(hk + 1) * rep].float().cpu().numpy().astype(np.float64)[None]
        ref = oracle.decode_attention(self.kp, self.vp, self.off, qn, kcodes, vcodes, [T],
                                      1.0 / math.sqrt(D))[0]
        parity.assert_close(out[b, hk * rep:(hk + 1) * rep].cpu().numpy(), ref, label)


def test_llama_layer_32k_sampled_heads():
    w = W.LLAMA_DECODE
    T = w.context
    K, V = _gen_kv(w, T, 0)
    cache = Cache(w, 1, T)
    cache.write(K, V, 0)
    g = torch.Generator(device=DEV)
    g.manual_seed(1)
    q = torch.randn((1, w.q_heads, w.head_dim), generator=g, device=DEV).to(torch.bfloat16)
    out = cache.decode(q, [T])
    torch.cuda.synchronize()
    assert cache.kctx[0].device_error() == 0
    for hk in (0, 5):
        cache.check_head(K, V, q, out, 0, hk, T, "llama hk=%d" % hk)


def test_serving_3p5bit_append_then_decode():
    """Batch 64 at 8192 tokens, groups 4 + 3 bits: prefill T-1 tokens, append one token per
    sequence (64 sequences x 8 kv heads) through scattered slots, then decode."""
    w = W.SERVING_3P5
    T = w.context
    K, V = _gen_kv(w, T, 3)
    cache = Cache(w, w.batch, T)
    cache.write(K[:, :, :T - 1], V[:, :, :T - 1], 0)
    cache.write(K[:, :, T - 1:], V[:, :, T - 1:], T - 1)          # the append step
    g = torch.Generator(device=DEV)
    g.manual_seed(4)
    q = torch.randn((w.batch, w.q_heads, w.head_dim), generator=g, device=DEV).to(torch.bfloat16)
    out = cache.decode(q, [T] * w.batch)
    torch.cuda.synchronize()
    for b, hk in ((0, 0), (37, 6), (63, 7)):
        cache.check_head(K, V, q, out, b, hk, T, "serving b=%d hk=%d" % (b, hk))


def test_long_context_2p5bit_decode_steps():
    """131072-token prefill at 2.5 bits (groups 3 + 2 bits), then decode steps that each
    append one token."""
    w = W.LONG_2P5
    T = w.context
    steps = 3
    K, V = _gen_kv(w, T + steps, 5)
    cache = Cache(w, 1, T + 32)
    cache.write(K[:, :, :T], V[:, :, :T], 0)
    g = torch.Generator(device=DEV)
    g.manual_seed(6)
    for s in range(steps):
        if s > 0:
            cache.write(K[:, :, T + s - 1:T + s], V[:, :, T + s - 1:T + s], T + s - 1)
        q = torch.randn((1, w.q_heads, w.head_dim), generator=g, device=DEV).to(torch.bfloat16)
        out = cache.decode(q, [T + s])
    torch.cuda.synchronize()
    cache.check_head(K, V, q, out, 0, 2, T + steps - 1, "long hk=2")


def _search_check(d, N, nq_sample, k=10, chunk=20000):
    """Full-size search on the GPU against the float64 estimator, query by query.

    For every sampled query: (1) the oracle's estimate of each returned id equals the
    returned score (elementwise, at the logit tolerance); (2) the returned ids are distinct
    and ordered by score, ties to the lower id; (3) the returned set is the oracle's top-k,
    except for ids whose oracle score lies within 2x tolerance of the oracle's k-th score
    (near-ties may swap); (4) 1@k recall against the exact float64 maximum inner product
    equals the oracle's, except on queries with such a near-tie.  The estimator oracle runs
    on the GPU's codes; the codes themselves are checked against the oracle's quantizer on
    a sample of database rows."""
    db = torch.nn.functional.normalize(torch.randn((N, d), generator=torch.Generator(device=DEV).manual_seed(7),
                                                   device=DEV), dim=1)
    qs = torch.nn.functional.normalize(torch.randn((1000, d), generator=torch.Generator(device=DEV).manual_seed(8),
                                                   device=DEV), dim=1)
    ctx = tq.Context(d, 4, 12, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, N)
    tq.quantize_kv(ctx, db, pk)
    scores, ids = tq.search_topk(ctx, qs, pk, N, k)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    op = oracle.make_params(d, 4, 12, 0)
    # quantizer parity on database rows spread over the whole range (first, last, strided)
    rows = torch.tensor(np.unique(np.r_[0, N - 1, np.linspace(0, N - 1, 254).astype(np.int64)]), device=DEV)
    parity.check_codes(op, db[rows].cpu().numpy().astype(np.float64), pk.codes[rows].cpu().numpy(),
                       pk.norm[rows].float().cpu().numpy(), pk.rnorm[rows].float().cpu().numpy(),
                       "search index d=%d" % d)
    sample = np.linspace(0, 999, nq_sample).astype(int)
    qn = qs[torch.tensor(sample, device=DEV)].cpu().numpy().astype(np.float64)
    s_gpu, i_gpu = scores.cpu().numpy().astype(np.float64), ids.cpu().numpy()
    # oracle estimates over the whole database (from the GPU's codes), chunk by chunk: the
    # k+1 best (score, id) per query, and the estimate of every returned id
    best = [[] for _ in sample]
    est_of_ret = np.full((len(sample), k), np.nan)
    exact_best = np.full(len(sample), -np.inf)
    exact_arg = np.zeros(len(sample), dtype=np.int64)
    for c0 in range(0, N, chunk):
        c1 = min(N, c0 + chunk)
        codes = pk.codes[c0:c1].cpu().numpy()
        cd = parity.codes_dict(codes, pk.norm[c0:c1].float().cpu().numpy(), pk.rnorm[c0:c1].float().cpu().numpy(),
                               d, 3, True)
        est = oracle.estimate_inner_products(op, qn, cd)
        for a, qi in enumerate(sample):
            top = np.argsort(-est[a], kind="stable")[:k + 1]
            best[a].extend([(-est[a][j], c0 + j) for j in top])
            inside = (i_gpu[qi] >= c0) & (i_gpu[qi] < c1)
            est_of_ret[a, inside] = est[a, i_gpu[qi][inside] - c0]
        ip = qn @ db[c0:c1].cpu().numpy().astype(np.float64).T
        arg = np.argmax(ip, axis=1)
        better = ip[np.arange(len(sample)), arg] > exact_best
        exact_best = np.where(better, ip[np.arange(len(sample)), arg], exact_best)
        exact_arg = np.where(better, c0 + arg, exact_arg)
    hits_gpu = hits_ref = 0
    for a, qi in enumerate(sample):
        lab = "search d=%d query %d" % (d, qi)
        ret = i_gpu[qi]
        assert len(set(ret.tolist())) == k and ret.min() >= 0 and ret.max() < N, lab + ": bad ids %s" % ret
        assert np.all(np.diff(s_gpu[qi]) <= 0), lab + ": scores not descending"
        ties = np.diff(s_gpu[qi]) == 0
        assert np.all(ret[1:][ties] > ret[:-1][ties]), lab + ": equal scores not in id order"
        parity.assert_close(s_gpu[qi], est_of_ret[a], lab + " (oracle estimate of each returned id)")
        ref = sorted(best[a])[:k + 1]
        ref_s = np.array([-x for x, _ in ref])
        ref_i = [j for _, j in ref]
        parity.assert_close(s_gpu[qi], ref_s[:k], lab + " (sorted top-k scores)")
        band = 2 * (parity.ATOL + parity.RTOL * abs(ref_s[k - 1]))
        near_tie = ref_s[k - 1] - ref_s[k] < band
        sure = {j for j, s in zip(ref_i[:k], ref_s[:k]) if s > ref_s[k - 1] + band}
        assert sure <= set(ret.tolist()), lab + ": missing oracle top-k ids %s" % sorted(sure - set(ret.tolist()))
        assert np.all(est_of_ret[a] >= ref_s[k - 1] - band), lab + ": returned id far below the oracle's k-th"
        h_g = int(exact_arg[a] in set(ret.tolist()))
        h_r = int(exact_arg[a] in set(ref_i[:k]))
        if not near_tie:
            assert set(ret.tolist()) == set(ref_i[:k]), lab + ": top-k set differs without a near-tie"
            assert h_g == h_r, lab + ": recall differs without a near-tie"
        hits_gpu += h_g
        hits_ref += h_r
    return hits_gpu / len(sample), hits_ref / len(sample)


def test_search_d200_one_million():
    r = _search_check(200, 1_000_000, 8)
    print("1@10 recall (sampled) d=200: gpu %.3f oracle %.3f" % r)


def test_search_d1536_one_million():
    r = _search_check(1536, 1_000_000, 8)
    print("1@10 recall (sampled) d=1536: gpu %.3f oracle %.3f" % r)
