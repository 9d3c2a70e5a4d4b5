"""CUDA path vs float64 oracle, element by element, through the C ABI (needs a B200)."""
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


def _bf16_rows(n, d, seed, outliers=False):
    x = W.gaussian((n, d), seed, W.STREAM_KEYS)
    if outliers:
        x[:, [3, 17, 60, 101][: max(1, d // 32)]] *= 8.0
    return W.round_bf16(x)


def _quantize(ctx, x_np, dtype, slots=None, cap=None):
    n = x_np.shape[0]
    x = torch.tensor(x_np, dtype=dtype, device=DEV)
    pk = tq.alloc_packed(ctx, cap or n)
    s = None if slots is None else torch.tensor(slots, dtype=torch.int64, device=DEV)
    tq.quantize_kv(ctx, x, pk, slots=s)
    torch.cuda.synchronize()
    return pk


def _host(pk, rows=None):
    sel = slice(None) if rows is None else torch.tensor(rows, device=DEV)
    codes = pk.codes[sel].cpu().numpy()
    norm = pk.norm[sel].float().cpu().numpy()
    rn = None if pk.rnorm is None else pk.rnorm[sel].float().cpu().numpy()
    return codes, norm, rn


# ------------------------------------------------------------------------------ params
@pytest.mark.parametrize("d,bits,mode", [(128, 4, 0), (64, 3, 1), (1536, 4, 0)])
def test_device_context_params_match_oracle(d, bits, mode):
    ctx = tq.Context(d, bits, 1000 + bits, mode)
    p = ctx.params()
    o = oracle.make_params(d, bits, 1000 + bits, mode)
    assert np.abs(p["Pi"] - o["Pi"]).max() < 1e-10
    assert np.abs(p["centroids"] - o["centroids"]).max() < 1e-10
    assert (ctx.d_pad, ctx.planes, ctx.code_bytes) == layout.geometry(d, o["k"], mode == 0)


# ---------------------------------------------------------------------------- quantize
def test_quantize_toy_config_fp32():
    """Keys N=4096 x 128 fp32 N(0,1) from seed 0, b = 3 (2-bit MSE + 1-bit QJL, m = 128)."""
    keys, _ = W.toy_inputs(0)
    ctx = tq.Context(128, 3, 1000, tq.MODE_PROD)
    pk = _quantize(ctx, keys, torch.float32)
    codes, norm, rn = _host(pk)
    res = parity.check_codes(oracle.make_params(128, 3, 1000, 0), keys.astype(np.float64), codes, norm, rn, "toy")
    print("toy quantize", res)


@pytest.mark.parametrize("d,bits,mode,n,dtype", [
    (128, 4, 0, 3000, "bf16"), (128, 4, 1, 3000, "bf16"),      # Llama-shaped keys / values
    (64, 4, 0, 1031, "bf16"), (64, 3, 0, 1031, "bf16"), (64, 2, 0, 517, "bf16"),
    (64, 4, 1, 1031, "bf16"), (64, 3, 1, 1031, "bf16"), (64, 2, 1, 517, "bf16"),
    (128, 5, 0, 300, "f16"), (128, 1, 1, 300, "fp32"),
    (200, 4, 0, 257, "fp32"), (1536, 4, 0, 65, "fp32"), (16, 3, 0, 129, "fp32"),
    (128, 4, 0, 1, "bf16"), (128, 4, 0, 127, "bf16"), (128, 4, 0, 129, "bf16"),
    (128, 2, 0, 700, "bf16"), (128, 3, 1, 700, "bf16"), (128, 2, 1, 700, "bf16"),   # tensor-core variants
    (64, 2, 1, 300, "bf16"), (128, 4, 0, 40000, "bf16"), (64, 4, 1, 40000, "bf16"),  # many tiles per CTA
    (128, 4, 1, 40000, "bf16"), (64, 3, 0, 40000, "bf16"), (128, 2, 0, 38000, "bf16"),
    (64, 2, 0, 40000, "bf16"), (64, 3, 1, 40001, "bf16"), (64, 2, 1, 39999, "bf16"),   # d = 64 shared words
    # workspace path: fp32 / fp16 input, every width, several N blocks, tiny batches
    (1536, 4, 0, 300, "fp32"), (200, 4, 0, 3000, "fp32"), (128, 3, 0, 4096, "fp32"),
    (3072, 4, 0, 40, "fp32"), (300, 3, 1, 257, "fp32"), (100, 2, 0, 129, "f16"),
    (64, 4, 1, 5, "bf16"), (128, 3, 0, 2, "bf16"), (32, 5, 0, 300, "fp32"), (3, 2, 1, 64, "fp32"),
])
def test_quantize_matches_oracle(d, bits, mode, n, dtype):
    seed = 1000 + 2 * bits + mode
    if dtype == "fp32":
        x = W.unit_gaussian(n, d, 3, 11) * 3.0
    else:
        x = _bf16_rows(n, d, 5, outliers=True)
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "fp32": torch.float32}[dtype]
    if dtype == "f16":
        x = x.astype(np.float16).astype(np.float32)
    ctx = tq.Context(d, bits, seed, mode)
    pk = _quantize(ctx, x, tdt)
    codes, norm, rn = _host(pk)
    res = parity.check_codes(oracle.make_params(d, bits, seed, mode), x.astype(np.float64), codes, norm, rn,
                             "d=%d b=%d mode=%d" % (d, bits, mode))
    assert ctx.device_error() == 0
    print(d, bits, mode, n, res)


def test_quantize_workspace_chunks_and_slots():
    """More rows than one workspace chunk (131072), fp32 input, scattered slots; rows in
    every chunk are compared with the oracle."""
    d, n, cap = 64, 140000, 150000
    x = (W.unit_gaussian(n, d, 5, 12) * 2.5).astype(np.float32)
    x[[0, 131071, 131072, 139999]] = 0.0
    rng = np.random.default_rng(9)
    slots = rng.permutation(cap)[:n]
    ctx = tq.Context(d, 4, 1010, tq.MODE_PROD)
    pk = _quantize(ctx, x, torch.float32, slots=slots, cap=cap)
    rows = np.r_[0:300, 131000:131400, 139700:140000]
    codes, norm, rn = _host(pk, rows=slots[rows])
    parity.check_codes(oracle.make_params(d, 4, 1010, 0), x[rows].astype(np.float64), codes, norm, rn, "chunks")
    assert ctx.device_error() == 0


def test_quantize_zero_rows_and_scattered_slots():
    d, n = 128, 300
    x = _bf16_rows(n, d, 9)
    x[[0, 17, 299]] = 0.0
    rng = np.random.default_rng(4)
    slots = rng.permutation(1000)[:n]
    ctx = tq.Context(d, 4, 77, tq.MODE_PROD)
    pk = _quantize(ctx, x, torch.bfloat16, slots=slots, cap=1000)
    codes, norm, rn = _host(pk, rows=slots)
    parity.check_codes(oracle.make_params(d, 4, 77, 0), x.astype(np.float64), codes, norm, rn, "zero+slots")
    assert norm[0] == 0 and rn[0] == 0
    # slots that were not written stay zero
    untouched = np.setdiff1d(np.arange(1000), slots)
    assert pk.codes[torch.tensor(untouched, device=DEV)].abs().sum().item() == 0


def test_quantize_strided_channel_group():
    """A group's channels are a slice of wider rows: x + offset, ld = row width."""
    full = _bf16_rows(500, 128, 13)
    xt = torch.tensor(full, dtype=torch.bfloat16, device=DEV)
    ctx = tq.Context(64, 3, 1003, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, 500)
    tq.quantize_kv(ctx, xt[:, 64:], pk)
    torch.cuda.synchronize()
    codes, norm, rn = _host(pk)
    parity.check_codes(oracle.make_params(64, 3, 1003, 0), full[:, 64:].astype(np.float64), codes, norm, rn, "slice")


# -------------------------------------------------------------------------- dequantize
def _dequant_ref(ctx, pk, d, bits, mode, seed, rows=None):
    codes, norm, rn = _host(pk, rows)
    cd = parity.codes_dict(codes, norm, rn, d, ctx.k, mode == 0)
    return oracle.dequantize(oracle.make_params(d, bits, seed, mode), cd["idx"], cd["norm"])


@pytest.mark.parametrize("d,bits,mode,n", [
    (128, 4, 1, 333), (128, 4, 0, 40000), (128, 3, 1, 4097), (128, 2, 0, 129),    # Llama-shaped, many tiles
    (64, 3, 0, 333), (64, 2, 1, 1000), (64, 4, 1, 256),                           # channel groups
    (100, 3, 1, 257), (96, 4, 0, 131), (32, 2, 1, 5), (16, 3, 0, 3),             # padded K / N, tiny n
    (128, 1, 1, 300), (128, 5, 0, 300), (48, 1, 1, 70),                           # 1-bit and 5-bit codes
])
def test_dequantize_matches_oracle(d, bits, mode, n):
    """x_hat = ||x|| Pi^T c[idx] of the stored codes on the tensor cores vs the float64
    definition applied to the same codes."""
    x = _bf16_rows(n, d, 21, outliers=True)
    seed = 5 + bits
    ctx = tq.Context(d, bits, seed, mode)
    pk = _quantize(ctx, x, torch.bfloat16)
    out = tq.dequantize(ctx, pk, n)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    parity.assert_close(out.cpu().numpy(), _dequant_ref(ctx, pk, d, bits, mode, seed), "dequant d=%d b=%d" % (d, bits))


@pytest.mark.parametrize("d,bits,n", [(128, 4, 4097), (64, 3, 333), (100, 2, 257), (128, 5, 300), (32, 2, 7)])
def test_dequantize_qjl_matches_oracle(d, bits, n):
    """QJL-augmented reconstruction x_hat = n (Pi^T c[idx] + sqrt(pi/2)/m r S^T (2s-1)) of
    the stored keys vs the float64 definition on the same codes."""
    x = _bf16_rows(n, d, 25, outliers=True)
    seed = 40 + bits
    ctx = tq.Context(d, bits, seed, tq.MODE_PROD)
    pk = _quantize(ctx, x, torch.bfloat16)
    out = tq.dequantize(ctx, pk, n, qjl=True)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    codes, norm, rn = _host(pk)
    cd = parity.codes_dict(codes, norm, rn, d, ctx.k, True)
    ref = oracle.dequantize_qjl(oracle.make_params(d, bits, seed, 0), cd["idx"], cd["signs"], cd["norm"], cd["rnorm"])
    parity.assert_close(out.cpu().numpy(), ref, "qjl dequant d=%d b=%d" % (d, bits))
    # the plain reconstruction of the same codes is unchanged by the QJL mode
    plain = tq.dequantize(ctx, pk, n).cpu().numpy()
    parity.assert_close(plain, oracle.dequantize(oracle.make_params(d, bits, seed, 0), cd["idx"], cd["norm"]), "plain")


def test_dequantize_gathered_slots_zero_rows_and_strided_output():
    """Slots gathered in any order, zero vectors, and an output that is a column slice of a
    wider fp32 tensor (row stride above d, start not 16-byte aligned)."""
    d, n, cap = 128, 700, 2000
    x = _bf16_rows(n, d, 23)
    x[[0, 350, 699]] = 0.0
    rng = np.random.default_rng(8)
    slots = rng.permutation(cap)[:n]
    ctx = tq.Context(d, 4, 31, tq.MODE_MSE)
    pk = _quantize(ctx, x, torch.bfloat16, slots=slots, cap=cap)
    gather = rng.permutation(slots)[:517]
    wide = torch.full((517, 3 + d + 5), 7.0, dtype=torch.float32, device=DEV)
    out = wide[:, 3:3 + d]
    tq.dequantize(ctx, pk, slots=torch.tensor(gather, dtype=torch.int64, device=DEV), out=out)
    torch.cuda.synchronize()
    ref = _dequant_ref(ctx, pk, d, 4, 1, 31, rows=gather)
    parity.assert_close(out.cpu().numpy(), ref, "dequant gathered")
    assert (wide[:, :3] == 7.0).all() and (wide[:, 3 + d:] == 7.0).all()   # nothing outside the slice
    zero_rows = np.isin(gather, slots[[0, 350, 699]])
    assert np.all(out.cpu().numpy()[zero_rows] == 0.0)


def test_dequantize_empty_and_unsupported_width():
    ctx = tq.Context(128, 4, 5, tq.MODE_MSE)
    pk = tq.alloc_packed(ctx, 4)
    out = torch.empty((0, 128), dtype=torch.float32, device=DEV)
    tq.dequantize(ctx, pk, 0, out=out)                    # nothing to do
    wide = tq.Context(200, 4, 5, tq.MODE_MSE)
    with pytest.raises(tq.TQError) as e:
        tq.dequantize(wide, tq.alloc_packed(wide, 4), 4)
    assert e.value.status == 2                             # TQ_ERR_UNSUPPORTED (d above 128)


def test_logits_toy_config():
    """16 queries x 4096 keys: logits from the GPU codes vs the oracle estimator on the
    same codes, and vs the oracle's end-to-end quantize + estimate."""
    keys, queries = W.toy_inputs(0)
    op = oracle.make_params(128, 3, 1000, 0)
    ctx = tq.Context(128, 3, 1000, tq.MODE_PROD)
    pk = _quantize(ctx, keys, torch.float32)
    q = torch.tensor(queries, device=DEV)
    lg = tq.attn_logits(ctx, q, pk, 4096).cpu().numpy()
    codes, norm, rn = _host(pk)
    ref = oracle.estimate_inner_products(op, queries.astype(np.float64), parity.codes_dict(codes, norm, rn, 128, 2, True))
    parity.assert_close(lg, ref, "logits(gpu codes)")
    rec = parity.reconciled_oracle_codes(op, keys.astype(np.float64), codes)
    assert rec["rows_reconciled"] <= 4
    e2e = oracle.estimate_inner_products(op, queries.astype(np.float64), rec)
    parity.assert_close(lg, e2e, "logits(end to end)")


@pytest.mark.parametrize("d,bits,n,nq", [(128, 4, 1000, 3), (64, 2, 777, 9), (64, 4, 300, 5), (128, 3, 1, 1)])
def test_logits_on_oracle_codes(d, bits, n, nq):
    """Codes produced by the oracle, packed on the host and uploaded: isolates the logits
    kernel from the quantizer."""
    op = oracle.make_params(d, bits, 31, 0)
    x = _bf16_rows(n, d, 2).astype(np.float64)
    o = oracle.quantize(op, x)
    codes = layout.pack(o["idx"], o["signs"], d, op["k"])
    ctx = tq.Context(d, bits, 31, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, n)
    pk.codes.copy_(torch.tensor(codes, device=DEV))
    pk.norm.copy_(torch.tensor(o["norm"], dtype=torch.float16, device=DEV))
    pk.rnorm.copy_(torch.tensor(o["rnorm"], dtype=torch.float16, device=DEV))
    qn = W.gaussian((nq, d), 8, W.STREAM_QUERIES).astype(np.float32)
    lg = tq.attn_logits(ctx, torch.tensor(qn, device=DEV), pk, n).cpu().numpy()
    parity.assert_close(lg, oracle.estimate_inner_products(op, qn.astype(np.float64), o), "logits")


@pytest.mark.parametrize("d,nq", [(128, 7), (64, 1), (200, 33), (300, 16), (1536, 5)])
def test_prepare_queries(d, nq):
    """Pi q and S q of unit-variance queries: chunks of 128 terms, ragged query and output
    blocks (d not a multiple of 16 or 128)."""
    ctx = tq.Context(d, 4, 3, tq.MODE_PROD)
    q = W.gaussian((nq, d), 1, 2).astype(np.float32)
    out = tq.prepare_queries(ctx, torch.tensor(q, device=DEV)).cpu().numpy()
    qt, qs = oracle.prepare_query(oracle.make_params(d, 4, 3, 0), q.astype(np.float64))
    tol = 1e-4 * np.sqrt(d / 128.0)
    assert np.abs(out[:, :d] - qt).max() < tol
    assert np.abs(out[:, d:] - qs).max() < 10 * tol


# ------------------------------------------------------------------------------ decode
def _decode_case(B, Hkv, Hq, D, groups, seq_lens, max_len, seed, q_dtype=torch.bfloat16):
    rng = np.random.default_rng(seed)
    K = W.round_bf16(rng.standard_normal((B, Hkv, max_len, D)))
    V = W.round_bf16(rng.standard_normal((B, Hkv, max_len, D)) * rng.lognormal(0, 0.5, (B, 1, max_len, 1)))
    qn = W.round_bf16(rng.standard_normal((B, Hq, D)))
    kctx, vctx, kc, vc, kp, vp, offs = [], [], [], [], [], [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        kx = tq.Context(w, kb, 1000 + 2 * gi, tq.MODE_PROD)
        vx = tq.Context(w, vb, 1001 + 2 * gi, tq.MODE_MSE)
        kpk = tq.alloc_packed(kx, B * Hkv * max_len)
        vpk = tq.alloc_packed(vx, B * Hkv * max_len)
        # prefill: token t of (b, h) -> slot (b*Hkv + h)*max_len + t, only t < seq_len
        rows, slots = [], []
        for b in range(B):
            for h in range(Hkv):
                for t in range(seq_lens[b]):
                    rows.append((b, h, t))
                    slots.append((b * Hkv + h) * max_len + t)
        if rows:
            ridx = np.array(rows)
            st = torch.tensor(slots, dtype=torch.int64, device=DEV)
            kr = torch.tensor(K[ridx[:, 0], ridx[:, 1], ridx[:, 2]][:, off:off + w].copy(), dtype=torch.bfloat16, device=DEV)
            vr = torch.tensor(V[ridx[:, 0], ridx[:, 1], ridx[:, 2]][:, off:off + w].copy(), dtype=torch.bfloat16, device=DEV)
            tq.quantize_kv(kx, kr, kpk, slots=st)
            tq.quantize_kv(vx, vr, vpk, slots=st)
        kctx.append(kx); vctx.append(vx); kc.append(kpk); vc.append(vpk)
        kp.append(oracle.make_params(w, kb, 1000 + 2 * gi, 0))
        vp.append(oracle.make_params(w, vb, 1001 + 2 * gi, 1))
        offs.append(off)
    offs.append(D)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    q = torch.tensor(qn, dtype=q_dtype, device=DEV)
    scale = 1.0 / math.sqrt(D)
    out = tq.decode_attention(kctx, vctx, offs, q, kc, vc, sl, Hkv, max_len, scale).cpu().numpy()
    # oracle on the GPU's stored codes
    kcodes, vcodes = [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        c, n_, r_ = _host(kc[gi])
        d1 = parity.codes_dict(c, n_, r_, w, kb - 1, True)
        kcodes.append({k: (None if v is None else v.reshape(B, Hkv, max_len, *v.shape[1:])) for k, v in d1.items()})
        c, n_, _ = _host(vc[gi])
        d2 = parity.codes_dict(c, n_, None, w, vb, False)
        vcodes.append({k: v.reshape(B, Hkv, max_len, *v.shape[1:]) for k, v in d2.items() if v is not None})
    ref = oracle.decode_attention(kp, vp, offs, qn.astype(np.float64), kcodes, vcodes, seq_lens, scale)
    _decode_case.last_caches = (kc, vc)
    return out, ref, (K, V, qn, kp, vp, offs)


@pytest.mark.parametrize("groups", [((0, 128, 4, 4),), ((0, 64, 4, 4), (64, 64, 3, 3)), ((0, 64, 3, 3), (64, 64, 2, 2))])
def test_decode_matches_oracle(groups):
    out, ref, _ = _decode_case(2, 2, 8, 128, groups, [300, 37], 320, 1)
    parity.assert_close(out, ref, "decode %s" % (groups,))


@pytest.mark.parametrize("groups", [((0, 128, 4, 4),), ((0, 64, 4, 4), (64, 64, 3, 3))])
def test_decode_odd_max_len(groups):
    """An odd cache length per (sequence, kv head): half of the caches start at an odd slot,
    so their staged code and norm arrays land at odd offsets inside the stage buffers."""
    out, ref, _ = _decode_case(2, 3, 12, 128, groups, [257, 130], 257, 21)
    parity.assert_close(out, ref, "decode odd max_len %s" % (groups,))


def test_decode_edge_lengths():
    """Empty sequence -> zeros; single token -> that token's dequantized value; ragged tails."""
    out, ref, (K, V, qn, kp, vp, offs) = _decode_case(4, 1, 4, 128, ((0, 128, 4, 4),), [0, 1, 129, 255], 256, 2)
    assert np.all(out[0] == 0.0)
    parity.assert_close(out, ref, "edge")


def test_decode_end_to_end_matches_oracle_pipeline():
    """GPU quantize + decode vs oracle quantize + decode on the same bf16 inputs."""
    groups = ((0, 128, 4, 4),)
    B, Hkv, Hq, D, T = 1, 2, 8, 128, 200
    out, _, (K, V, qn, kp, vp, offs) = _decode_case(B, Hkv, Hq, D, groups, [T], T, 3)
    kg, vg = _decode_case.last_caches
    ko = parity.reconciled_oracle_codes(kp[0], K.reshape(-1, D).astype(np.float64), _host(kg[0])[0])
    vo = parity.reconciled_oracle_codes(vp[0], V.reshape(-1, D).astype(np.float64), _host(vg[0])[0])
    kcodes = [{k: (None if v is None else v.reshape(B, Hkv, T, *v.shape[1:])) for k, v in
               dict(idx=ko["idx"], norm=ko["norm"], signs=ko["signs"], rnorm=ko["rnorm"]).items()}]
    vcodes = [dict(idx=vo["idx"].reshape(B, Hkv, T, D), norm=vo["norm"].reshape(B, Hkv, T))]
    ref = oracle.decode_attention(kp, vp, offs, qn.astype(np.float64), kcodes, vcodes, [T], 1 / math.sqrt(D))
    parity.assert_close(out, ref, "e2e decode")


# ------------------------------------------------------------------------------ search
@pytest.mark.parametrize("d,N,k,bits,nq", [
    (128, 5000, 10, 4, 6), (200, 3000, 10, 4, 6), (64, 100, 64, 4, 6),     # 4-bit codes (byte-permute decode)
    (1536, 3000, 10, 4, 6), (3072, 700, 5, 4, 3), (96, 513, 33, 4, 6),     # wide / ragged chunk
    (128, 2000, 10, 4, 300), (128, 300, 1, 4, 129),                        # several query tiles
    (128, 2000, 10, 2, 6), (100, 1500, 7, 3, 6), (160, 1200, 10, 5, 6),    # 1-, 2-, 4-bit indices
    (64, 900, 32, 4, 6),                                                   # largest k with two lists per query
])
def test_search_topk_matches_oracle(d, N, k, bits, nq):
    db = W.unit_gaussian(N, d, 1, 10)
    db[N // 2] = db[7]                        # an exact tie: lower id must come first
    qs = W.unit_gaussian(nq, d, 1, 3)
    qs[0] = db[7]
    ctx = tq.Context(d, bits, 12, tq.MODE_PROD)
    pk = _quantize(ctx, db, torch.float32)
    scores, ids = tq.search_topk(ctx, torch.tensor(qs, device=DEV), pk, N, k)
    scores, ids = scores.cpu().numpy(), ids.cpu().numpy()
    assert ctx.device_error() == 0
    codes, norm, rn = _host(pk)
    op = oracle.make_params(d, bits, 12, 0)
    cd = parity.codes_dict(codes, norm, rn, d, bits - 1, True)
    est = oracle.estimate_inner_products(op, qs.astype(np.float64), cd)
    ref_s, ref_i = oracle.search_topk(op, qs.astype(np.float64), cd, k)
    parity.assert_close(scores, ref_s, "top-k scores")
    for a in range(len(qs)):
        assert len(set(ids[a])) == k
        parity.assert_close(scores[a], est[a, ids[a]], "score of returned id")
        # ids agree wherever the oracle's scores are separated by more than the tolerance
        gap = np.abs(np.diff(np.sort(est[a])[::-1][: k + 1]))
        if gap.min() > 2 * (parity.ATOL + parity.RTOL * np.abs(ref_s[a]).max()):
            assert list(ids[a]) == list(ref_i[a])
    row = list(ids[0])
    if 7 in row and N // 2 in row and scores[0][row.index(7)] == scores[0][row.index(N // 2)]:
        assert row.index(7) < row.index(N // 2)        # equal scores: lower id first


def test_decode_many_splits():
    """One kv head over 7000 tokens: 110 context splits of 64 tokens, so the merge stages the
    partials in two bulk-copy chunks (96 + 14 splits) and one query-prep block is ragged."""
    out, ref, _ = _decode_case(1, 1, 4, 128, ((0, 128, 4, 4),), [7000], 7040, 11)
    parity.assert_close(out, ref, "decode, 110 splits")


@pytest.mark.parametrize("Hkv,Hq", [(2, 4), (1, 8), (3, 12), (4, 4), (2, 12), (1, 16)])
def test_decode_other_gqa_ratios(Hkv, Hq):
    """Every GQA ratio on the tensor-core kernel: 1, 2, 4, 6, 8 and 16 query heads per kv
    head (a CTA serves 4 query heads of one kv head; ratios that are not a multiple of 4
    repeat a head in the spare MMA columns and drop its result)."""
    out, ref, _ = _decode_case(2, Hkv, Hq, 128, ((0, 128, 4, 4),), [100, 33], 128, 7)
    parity.assert_close(out, ref, "gqa %d/%d" % (Hq, Hkv))


def _perm_case(perm_kind, seed=11):
    """2.5-bit groups (64 ch at 3 + 3 bits, 64 ch at 2 + 2 bits) on data with 4 outlier
    channels x8 per kv head; channel_perm per kv head: "random", or "outlier" (the channels
    with the largest RMS over the sample first, so the outliers get the higher bit width)."""
    B, Hkv, Hq, D, T = 2, 2, 8, 128, 300
    groups = ((0, 64, 3, 3), (64, 64, 2, 2))
    rng = np.random.default_rng(seed)
    K = W.round_bf16(rng.standard_normal((B, Hkv, T, D)))
    V = W.round_bf16(rng.standard_normal((B, Hkv, T, D)))
    for h in range(Hkv):                          # outliers in the second (low-bit) half by default
        ch = 64 + rng.choice(64, 4, replace=False)
        K[:, h, :, ch] *= 8.0
        V[:, h, :, ch] *= 8.0
    K, V = W.round_bf16(K), W.round_bf16(V)
    q = W.round_bf16(rng.standard_normal((B, Hq, D)))
    if perm_kind == "random":
        perm = np.stack([rng.permutation(D) for _ in range(Hkv)]).astype(np.int32)
    elif perm_kind == "identity":
        perm = np.stack([np.arange(D)] * Hkv).astype(np.int32)
    else:
        perm = np.stack([tq.channel_perm_by_score(np.sqrt((K[:, h] ** 2).mean(axis=(0, 1))), 64)
                         for h in range(Hkv)]).astype(np.int32)
    kctx, vctx, kc, vc, kp, vp = [], [], [], [], [], []
    Kt = torch.tensor(K.reshape(-1, D), dtype=torch.bfloat16, device=DEV)
    Vt = torch.tensor(V.reshape(-1, D), dtype=torch.bfloat16, device=DEV)
    for gi, (off, w, kb, vb) in enumerate(groups):
        kx = tq.Context(w, kb, 1000 + 2 * gi, tq.MODE_PROD)
        vx = tq.Context(w, vb, 1001 + 2 * gi, tq.MODE_MSE)
        kpk, vpk = tq.alloc_packed(kx, B * Hkv * T), tq.alloc_packed(vx, B * Hkv * T)
        for h in range(Hkv):                      # rows of kv head h: its own columns
            rows = torch.tensor([(b * Hkv + h) * T + t for b in range(B) for t in range(T)], device=DEV)
            cols = torch.tensor(perm[h, off:off + w], dtype=torch.int32, device=DEV)
            tq.quantize_kv(kx, Kt[rows], kpk, slots=rows, cols=cols)
            tq.quantize_kv(vx, Vt[rows], vpk, slots=rows, cols=cols)
        kctx.append(kx); vctx.append(vx); kc.append(kpk); vc.append(vpk)
        kp.append(oracle.make_params(w, kb, 1000 + 2 * gi, 0)); vp.append(oracle.make_params(w, vb, 1001 + 2 * gi, 1))
    sl = torch.tensor([T, 171], dtype=torch.int32, device=DEV)
    out = tq.decode_attention(kctx, vctx, [0, 64, 128], torch.tensor(q, dtype=torch.bfloat16, device=DEV), kc, vc,
                              sl, Hkv, T, 1 / np.sqrt(D),
                              channel_perm=torch.tensor(perm, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    # the oracle's own codes of the permuted columns (reconciled with the GPU's on exempt choices)
    kcodes, vcodes = [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        kx_ = np.stack([K[:, h][..., perm[h, off:off + w]] for h in range(Hkv)], axis=1)
        vx_ = np.stack([V[:, h][..., perm[h, off:off + w]] for h in range(Hkv)], axis=1)
        ko = parity.reconciled_oracle_codes(kp[gi], kx_.reshape(-1, w).astype(np.float64), kc[gi].codes.cpu().numpy())
        vo = parity.reconciled_oracle_codes(vp[gi], vx_.reshape(-1, w).astype(np.float64), vc[gi].codes.cpu().numpy())
        kcodes.append({k: ko[k].reshape(B, Hkv, T, *ko[k].shape[1:]) for k in ("idx", "signs", "norm", "rnorm")})
        vcodes.append({k: vo[k].reshape(B, Hkv, T, *vo[k].shape[1:]) for k in ("idx", "norm")})
    ref = oracle.decode_attention(kp, vp, [0, 64, 128], q.astype(np.float64), kcodes, vcodes, [T, 171],
                                  1 / np.sqrt(D), channel_perm=perm)
    # exact attention on the unquantized inputs (for the quality comparison)
    exact = np.zeros_like(ref)
    for b, Tb in enumerate([T, 171]):
        for hq in range(Hq):
            h = hq // (Hq // Hkv)
            lg = K[b, h, :Tb].astype(np.float64) @ q[b, hq].astype(np.float64) / np.sqrt(D)
            p = np.exp(lg - lg.max())
            exact[b, hq] = (p / p.sum()) @ V[b, h, :Tb].astype(np.float64)
    return out.cpu().numpy(), ref, exact


@pytest.mark.parametrize("perm_kind", ["random", "outlier"])
def test_decode_channel_permutation_matches_oracle(perm_kind):
    out, ref, _ = _perm_case(perm_kind)
    parity.assert_close(out, ref, "decode with %s channel permutation" % perm_kind)


def test_outlier_aware_grouping_lowers_the_attention_error():
    """Sending the outlier channels to the higher-bit group, instead of leaving them in the
    2-bit half (the contiguous split), brings the quantized attention closer to exact
    attention on the same inputs."""
    out_o, _, exact = _perm_case("outlier")
    out_i, ref_i, exact_i = _perm_case("identity")
    assert np.array_equal(exact, exact_i)
    parity.assert_close(out_i, ref_i, "decode with the identity permutation")
    err_outlier = np.abs(out_o - exact).mean()
    err_default = np.abs(out_i - exact).mean()
    print("mean |attention - exact|: outlier-aware %.4g, contiguous %.4g" % (err_outlier, err_default))
    assert err_outlier < err_default


def test_unsupported_shapes_are_reported():
    """Shapes outside the tensor-core kernels return TQ_ERR_UNSUPPORTED (no slower path)."""
    ctx = tq.Context(200, 4, 3, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, 8)
    with pytest.raises(tq.TQError) as e:
        tq.attn_logits(ctx, torch.zeros((2, 200), device=DEV), pk, 8)
    assert e.value.status == 2
    kx, vx = tq.Context(64, 4, 1, tq.MODE_PROD), tq.Context(64, 4, 2, tq.MODE_MSE)
    kc, vc = tq.alloc_packed(kx, 2 * 16), tq.alloc_packed(vx, 2 * 16)
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device=DEV)
    sl = torch.tensor([16], dtype=torch.int32, device=DEV)
    with pytest.raises(tq.TQError) as e:
        tq.decode_attention([kx], [vx], [0, 64], q, [kc], [vc], sl, 2, 16, 0.125)
    assert e.value.status == 2


def test_decode_fp32_queries_and_128_2bit_keys():
    out, ref, _ = _decode_case(1, 2, 8, 128, ((0, 128, 3, 3),), [513], 600, 8, q_dtype=torch.float32)
    parity.assert_close(out, ref, "fp32 q, 3-bit keys / values")


# ------------------------------------------------------------- paged caches, one-graph steps
def _oracle_decode(groups, K, V, q, lens, D, kc_gpu, vc_gpu, max_len):
    """Oracle decode of K/V [B, Hkv, T, D] over the oracle's codes, reconciled with the GPU's
    exempt choices (codes of token t of (b, h) in slot (b*Hkv + h)*max_len + t of the given
    contiguous GPU caches)."""
    B, Hkv, T, _ = K.shape
    kp = [oracle.make_params(w, kb, 1000 + 2 * gi, 0) for gi, (_, w, kb, _) in enumerate(groups)]
    vp = [oracle.make_params(w, vb, 1001 + 2 * gi, 1) for gi, (_, w, _, vb) in enumerate(groups)]
    rows = torch.tensor([(b * Hkv + h) * max_len + t for b in range(B) for h in range(Hkv) for t in range(T)],
                        device=DEV)
    kc, vc = [], []
    for gi, (off, w, _, _) in enumerate(groups):
        ko = parity.reconciled_oracle_codes(kp[gi], K[..., off:off + w].reshape(-1, w).astype(np.float64),
                                            kc_gpu[gi].codes[rows].cpu().numpy())
        vo = parity.reconciled_oracle_codes(vp[gi], V[..., off:off + w].reshape(-1, w).astype(np.float64),
                                            vc_gpu[gi].codes[rows].cpu().numpy())
        kc.append({k: ko[k].reshape(B, Hkv, T, *ko[k].shape[1:]) for k in ("idx", "signs", "norm", "rnorm")})
        vc.append({k: vo[k].reshape(B, Hkv, T, *vo[k].shape[1:]) for k in ("idx", "norm")})
    offs = [g[0] for g in groups] + [D]
    return oracle.decode_attention(kp, vp, offs, q.astype(np.float64), kc, vc, lens, 1 / math.sqrt(D))


def test_paged_cache_decode_matches_contiguous_and_oracle():
    """A pool of 64-token pages in shuffled physical order (block table per sequence) gives
    the same attention as the contiguous cache, and both match the oracle."""
    groups = ((0, 64, 4, 4), (64, 64, 3, 3))
    B, Hkv, Hq, D, page, max_pages = 3, 2, 8, 128, 64, 5
    max_len = page * max_pages
    lens = [300, 129, 64]
    rng = np.random.default_rng(21)
    K = W.round_bf16(rng.standard_normal((B, Hkv, max_len, D)))
    V = W.round_bf16(rng.standard_normal((B, Hkv, max_len, D)))
    q = W.round_bf16(rng.standard_normal((B, Hq, D)))
    npool = B * max_pages + 2
    table = rng.permutation(npool)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    Kt = torch.tensor(K.reshape(-1, D), dtype=torch.bfloat16, device=DEV)
    Vt = torch.tensor(V.reshape(-1, D), dtype=torch.bfloat16, device=DEV)
    # slot of row (b, h, t) in the contiguous and in the paged cache
    b_, h_, t_ = np.meshgrid(np.arange(B), np.arange(Hkv), np.arange(max_len), indexing="ij")
    paged = (table[b_, t_ // page].astype(np.int64) * Hkv + h_) * page + t_ % page
    paged = torch.tensor(paged.reshape(-1), device=DEV)
    kx, vx, kc, vc, kpg, vpg = [], [], [], [], [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        a, b = tq.Context(w, kb, 1000 + 2 * gi, tq.MODE_PROD), tq.Context(w, vb, 1001 + 2 * gi, tq.MODE_MSE)
        kx.append(a); vx.append(b)
        kc.append(tq.alloc_packed(a, B * Hkv * max_len)); vc.append(tq.alloc_packed(b, B * Hkv * max_len))
        kpg.append(tq.alloc_packed(a, npool * Hkv * page)); vpg.append(tq.alloc_packed(b, npool * Hkv * page))
        tq.quantize_kv(a, Kt[:, off:off + w], kc[gi]); tq.quantize_kv(b, Vt[:, off:off + w], vc[gi])
        tq.quantize_kv(a, Kt[:, off:off + w], kpg[gi], slots=paged)
        tq.quantize_kv(b, Vt[:, off:off + w], vpg[gi], slots=paged)
    qt = torch.tensor(q, dtype=torch.bfloat16, device=DEV)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out_c = tq.decode_attention(kx, vx, [0, 64, 128], qt, kc, vc, sl, Hkv, max_len, 1 / math.sqrt(D))
    out_p = tq.decode_attention(kx, vx, [0, 64, 128], qt, kpg, vpg, sl, Hkv, max_len, 1 / math.sqrt(D),
                                block_table=torch.tensor(table, device=DEV), page_tokens=page)
    torch.cuda.synchronize()
    assert kx[0].device_error() == 0
    assert torch.equal(out_c, out_p)
    ref = _oracle_decode(groups, K, V, q, lens, D, kc, vc, max_len)
    parity.assert_close(out_p.cpu().numpy(), ref, "paged decode")


def test_append_and_decode_replayed_as_one_cuda_graph():
    """One CUDA graph holds a step's append-quantize (one new token per sequence and kv head,
    scattered slots) and its decode; the host only refreshes the graph's input buffers
    (new rows, slots, sequence lengths, query) between replays."""
    groups = ((0, 64, 4, 4), (64, 64, 3, 3))
    B, Hkv, Hq, D, T0, steps = 4, 2, 8, 128, 200, 3
    max_len = T0 + steps
    rng = np.random.default_rng(33)
    K = W.round_bf16(rng.standard_normal((B, Hkv, max_len, D)))
    V = W.round_bf16(rng.standard_normal((B, Hkv, max_len, D)))
    qs = W.round_bf16(rng.standard_normal((steps, B, Hq, D)))
    kx, vx, kc, vc = [], [], [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        a, b = tq.Context(w, kb, 1000 + 2 * gi, tq.MODE_PROD), tq.Context(w, vb, 1001 + 2 * gi, tq.MODE_MSE)
        kx.append(a); vx.append(b)
        kc.append(tq.alloc_packed(a, B * Hkv * max_len)); vc.append(tq.alloc_packed(b, B * Hkv * max_len))
    # prefill T0 tokens
    rows = torch.tensor([(bb * Hkv + h) * max_len + t for bb in range(B) for h in range(Hkv) for t in range(T0)],
                        device=DEV)
    Kt = torch.tensor(K.reshape(-1, D), dtype=torch.bfloat16, device=DEV)
    Vt = torch.tensor(V.reshape(-1, D), dtype=torch.bfloat16, device=DEV)
    for gi, (off, w, _, _) in enumerate(groups):
        tq.quantize_kv(kx[gi], Kt[rows, off:off + w], kc[gi], slots=rows)
        tq.quantize_kv(vx[gi], Vt[rows, off:off + w], vc[gi], slots=rows)
    # static graph inputs
    new_k = torch.zeros((B * Hkv, D), dtype=torch.bfloat16, device=DEV)
    new_v = torch.zeros_like(new_k)
    slots = torch.zeros(B * Hkv, dtype=torch.int64, device=DEV)
    seq = torch.zeros(B, dtype=torch.int32, device=DEV)
    qb = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((B, Hq, D), dtype=torch.float32, device=DEV)
    plan = tq.DecodePlan(kx, vx, [0, 64, 128], kc, vc, B, Hq, Hkv, D, max_len)
    # quantize workspaces sized once (the bf16 d = 64 rows of 8 tokens take the workspace path)
    wks = [torch.empty(max(tq.quantize_workspace_size(c, 1, B * Hkv, D), 1), dtype=torch.uint8, device=DEV)
           for c in kx + vx]

    def step():
        for gi, (off, w, _, _) in enumerate(groups):
            tq.quantize_kv(kx[gi], new_k[:, off:off + w], kc[gi], slots=slots, workspace=wks[gi])
            tq.quantize_kv(vx[gi], new_v[:, off:off + w], vc[gi], slots=slots, workspace=wks[len(groups) + gi])
        plan(qb, seq, 1 / math.sqrt(D), out)

    def load(s):
        t = T0 + s
        new_k.copy_(torch.tensor(K[:, :, t].reshape(-1, D), dtype=torch.bfloat16))
        new_v.copy_(torch.tensor(V[:, :, t].reshape(-1, D), dtype=torch.bfloat16))
        slots.copy_(torch.tensor([(bb * Hkv + h) * max_len + t for bb in range(B) for h in range(Hkv)]))
        seq.fill_(t + 1)
        qb.copy_(torch.tensor(qs[s], dtype=torch.bfloat16))

    load(0)
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        step()                                   # warm-up outside capture (first-use set-up)
    torch.cuda.current_stream().wait_stream(cs)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for s in range(steps):
        load(s)
        graph.replay()
        torch.cuda.synchronize()
        T = T0 + s + 1
        ref = _oracle_decode(groups, K[:, :, :T], V[:, :, :T], qs[s], [T] * B, D, kc, vc, max_len)
        parity.assert_close(out.cpu().numpy(), ref, "graph step %d" % s)
    assert kx[0].device_error() == 0
