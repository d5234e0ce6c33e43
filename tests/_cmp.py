"""Comparison helpers for GPU-vs-oracle parity (test code only).

Match criteria for the codec (written here once, used by every parity test):
  * E4M3 codes: bit-exact on >= 99.9 % of elements; every other element
    one code step away (adjacent representable values; +0 and -0 count as
    the same value).  The kernels form W in fp32 with a different summation
    order than the fp64 oracle, so a value within ~1e-6 of a rounding
    boundary may land on the neighbouring code.
  * scales: relative error <= 1e-3 (they are amax/448 of the same W).
  * G_hat (decoder fed the oracle's codes): fp32 output within 1e-3 of the
    oracle relative to the row's largest magnitude; bf16 output within one
    bf16 rounding (2^-8 relative) of the same reference plus that 1e-3.
    Each row also meets the criterion as a whole: its relative Frobenius
    error ||got - want|| / ||want|| is at most 1e-3 (plus 2^-8 for bf16
    output), so small elements cannot hide a large share of the error.
  * E4M3 under a dense transform (W = G M with a full-rank whitening M): the
    entries of M are large next to W (the sum cancels), so the fp32
    evaluation of W on the tensor cores carries an error that the codes
    resolve.  The criterion is derived from that arithmetic: with
    E_j = (K + 1) 2^-24 sum_i |G_i| |M_ij| (the deterministic bound of a
    K-term fp32 dot product, plus the 2^-24 of M's three bf16 parts), every
    decoded element lies within half an E4M3 step (at its own scale) plus E_j
    of the oracle's W, every scale within max_block(E) / 448 of the oracle's,
    and at least 99 % of the codes are exact.
  * NVFP4, Euclidean: every decision is taken in fp32 on exact inputs, so the
    tensor scale, block scales and codes are bit-exact (+0 / -0 the same).
  * NVFP4, whitened: W comes from the tensor cores (different summation
    order), so the tensor scale is within 1e-5 relative; block scale codes are
    exact on >= 99.9 % of blocks and one E4M3 step away elsewhere; inside
    blocks whose scale codes agree, E2M1 codes are exact on >= 99.9 % and one
    step away elsewhere.
"""
import numpy as np

CODE_EXACT_FRAC = 0.999
SCALE_RTOL = 1e-3
GHAT_RTOL = 1e-3


def e4m3_position(codes):
    c = np.asarray(codes, dtype=np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def check_codes(got, want, frac=CODE_EXACT_FRAC):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape
    exact = got == want
    pos_diff = np.abs(e4m3_position(got) - e4m3_position(want))
    same_value = pos_diff == 0  # +0 / -0
    ok = exact | same_value
    rate = ok.mean() if ok.size else 1.0
    assert rate >= frac, f"bit-exact rate {rate:.6f} < {frac}"
    assert pos_diff.max(initial=0) <= 1, f"max code distance {pos_diff.max()}"
    return rate


def check_scales(got, want, rtol=SCALE_RTOL):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want) / np.maximum(np.abs(want), 1e-300)
    err = np.where(want == 0, np.abs(got), err)
    assert err.max(initial=0) <= rtol, f"scale rel err {err.max()}"


def check_rows(got, want, rtol=GHAT_RTOL, bf16=False):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    rowmax = np.max(np.abs(want), axis=1, keepdims=True)
    tol = rtol * rowmax
    if bf16:
        tol = tol + 2.0 ** -8 * np.abs(want)
    bad = np.abs(got - want) > tol + 1e-30
    assert not bad.any(), f"{bad.sum()} elements off; worst {(np.abs(got - want) / np.maximum(rowmax, 1e-30)).max()}"
    rn = np.linalg.norm(want, axis=1)
    rel = np.linalg.norm(got - want, axis=1) / np.maximum(rn, 1e-300)
    rel = np.where(rn == 0, np.linalg.norm(got, axis=1), rel)
    lim = rtol + (2.0 ** -8 if bf16 else 0.0)
    assert rel.max(initial=0) <= lim, f"row relative Frobenius error {rel.max()} > {lim}"
    return float(rel.max(initial=0))


def e2m1_position(codes):
    c = np.asarray(codes, dtype=np.int64) & 0xF
    mag = c & 0x7
    return np.where(c & 0x8, -mag, mag)


def unpack_nibbles(packed):
    p = np.asarray(packed, dtype=np.uint8)
    q = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    q[:, 0::2] = p & 0xF
    q[:, 1::2] = p >> 4
    return q


def check_nvfp4(got, want, exact=False, frac=CODE_EXACT_FRAC, st_rtol=1e-5):
    """got / want: (packed codes, block scale codes, tensor scale)."""
    (gc, gs, gt), (wc, ws, wt) = got, want
    gt, wt = float(np.asarray(gt).reshape(-1)[0]), float(wt)
    qg, qw = e2m1_position(unpack_nibbles(gc)), e2m1_position(unpack_nibbles(wc))
    sg, sw = e4m3_position(gs), e4m3_position(ws)
    if exact:
        assert gt == wt, (gt, wt)
        assert np.array_equal(sg, sw), f"{(sg != sw).sum()} block scales differ"
        assert np.array_equal(qg, qw), f"{(qg != qw).sum()} codes differ"
        return
    assert abs(gt - wt) <= st_rtol * abs(wt), (gt, wt)
    ds = np.abs(sg - sw)
    assert ds.max(initial=0) <= 1 and (ds == 0).mean() >= frac, f"block scales: {(ds != 0).sum()} differ"
    same = np.repeat(ds == 0, 16, axis=1)
    dq = np.abs(qg - qw)[same]
    assert dq.max(initial=0) <= 1, f"max E2M1 code distance {dq.max()}"
    assert (dq == 0).mean() >= frac if dq.size else True, f"code exact rate {(dq == 0).mean():.6f}"


def check_codes_within_bound(codes, scales, W, E, min_exact_frac=0.99, want_codes=None, block=128):
    """Codes of W (fp64, oracle) under an error bound E (same shape) of the
    kernel's evaluation of W; see the module docstring.  Returns the exact
    rate against want_codes when given."""
    from oracle import gift_oracle as O
    codes = np.asarray(codes)
    W = np.asarray(W, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    d_out, d_in = W.shape
    s = np.repeat(np.asarray(scales, dtype=np.float64), block, axis=1)
    got = O.e4m3_decode(codes) * s
    y = (np.abs(W) + E) / np.where(s > 0, s, 1.0)
    step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3), 2.0 ** -9)
    allowed = 0.5 * step * s + E + 1e-30
    bad = np.abs(got - W) > allowed * (1 + 1e-9)
    assert not bad.any(), f"{bad.sum()} codes outside the bound; worst excess {(np.abs(got - W) / allowed).max()}"
    Eb = E.reshape(d_out, d_in // block, block).max(axis=2)
    Wb = np.abs(W).reshape(d_out, d_in // block, block).max(axis=2)
    ds = np.abs(np.asarray(scales, dtype=np.float64) - Wb / 448.0)
    assert np.all(ds <= Eb / 448.0 * (1 + 1e-6) + 1e-7 * Wb / 448.0), f"scale off by {ds.max()}"
    if want_codes is not None:
        rate = float((codes == np.asarray(want_codes)).mean())
        assert rate >= min_exact_frac, f"exact code rate {rate:.6f} < {min_exact_frac}"
        return rate
    return None
