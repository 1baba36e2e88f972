"""The fused kernel's certified selection window, checked on the CPU.

The fused kernel does not rank all M logits of a token.  Its steps:
1. Pass 1 reduces each 32-expert chunk to the maximum of its z_hi logits and packs it into an
   ordered 32-bit key, with the chunk id in the low bits.
2. It keeps the best k + 6 keys.
3. From the k-th key's value bits (rounded down) tlow and the bound eps on |z_hi logit - exact
   logit| (|z_lo| times the largest R2 column norm, by Cauchy-Schwarz, plus a rounding
   margin), it takes the chunks whose maxima can reach tlow - 2 eps and the experts in them
   whose exact logit reaches tlow - eps.
4. A list whose last key still reaches the cut goes to an exact fallback.

This test reimplements those steps in numpy (fp64 logits, fp32 keys, the same bit packing) and
checks the claim the kernel's exactness rests on: unless the token falls back, the exact top-k
(larger logit first, lower expert first on ties) is among the candidates.  It does so on
random, tie-heavy and near-tie inputs.  It tests the method's logic, not the CUDA code.
"""
import numpy as np
import pytest

import oracle
import synthetic as syn

KREAL = np.uint32(0x00800000)  # ordered value of -FLT_MAX: keys below name no real chunk


def ord_key(f32):
    b = np.asarray(f32, dtype=np.float32).view(np.uint32)
    return np.where(b >> 31, ~b, b | np.uint32(0x80000000)).astype(np.uint32)


def ord_inv(u):
    u = np.asarray(u, dtype=np.uint32)
    return np.where(u & np.uint32(0x80000000), u & np.uint32(0x7FFFFFFF), ~u).astype(np.uint32).view(np.float32)


def bf16_round(x):
    return syn.bf16_bits_to_f64(syn.f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def window(z, R2, k, KL):
    """Candidates of one token by the window rule; None when the token falls back."""
    r, M = R2.shape
    nchunks = 4 * ((M + 127) // 128)
    low = np.uint32((1 << int(np.ceil(np.log2(nchunks)))) - 1)
    z_hi = bf16_round(z)
    z_lo = bf16_round(z - z_hi)
    l_hi = z_hi @ R2
    exact = (z_hi + z_lo) @ R2
    padded = np.full(nchunks * 32, -np.inf)
    padded[:M] = l_hi
    cmax = np.sqrt((R2 * R2).sum(axis=0).max()) * (1 + 2.0 ** -20)
    keys = (ord_key(padded.reshape(nchunks, 32).max(axis=1).astype(np.float32)) & ~low) | np.arange(
        nchunks, dtype=np.uint32)
    keys = np.concatenate([np.sort(keys)[::-1], np.zeros(KL, np.uint32)])[:KL]  # unused slots hold key 0
    kth = keys[k - 1]
    valid = (keys & ~low) >= KREAL
    if (kth & ~low) < KREAL:  # fewer than k real chunks: every chunk is needed, no cut
        needed = keys[valid] & low
        cand = np.concatenate([np.arange(32 * c, min(32 * c + 32, M)) for c in needed])
        return cand, exact
    eps = np.linalg.norm(z_lo) * cmax * (1 + 2.0 ** -8) + r * 2.0 ** -20 * np.linalg.norm(z_hi) * cmax + 1e-30
    tlow = float(ord_inv(kth & ~low))
    ccut = tlow - eps
    cut_key = ord_key(np.float32(np.nextafter(np.float32(tlow - 2 * eps), np.float32(-np.inf))))
    if valid[-1] and (keys[-1] | low) >= cut_key:
        return None  # the list is too short to certify the cut
    needed = keys[valid & ((keys | low) >= cut_key)] & low
    cand = np.concatenate([np.arange(32 * c, min(32 * c + 32, M)) for c in needed]) if needed.size else np.array([], int)
    return cand[exact[cand] >= ccut], exact


def true_topk(exact, k):
    order = np.lexsort((np.arange(exact.size), -exact))
    return order[:k]


def check_tokens(Z, R2, k, KL):
    fallbacks = 0
    for z in Z:
        res = window(z, R2, k, KL)
        if res is None:
            fallbacks += 1
            continue
        cand, exact = res
        top = true_topk(exact, k)
        assert set(top.tolist()) <= set(cand.tolist()), "a top-k expert is outside the candidates"
        assert cand.size >= k
    return fallbacks


@pytest.mark.parametrize("N,h,r,M,k,unit", [(300, 128, 32, 192, 4, False), (300, 512, 32, 1024, 8, False),
                                             (200, 2048, 32, 4096, 8, True), (200, 256, 16, 256, 16, False),
                                             (200, 512, 64, 2048, 8, False)])
def test_window_holds_on_random_tokens(N, h, r, M, k, unit):
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=7, x_unit_rms=unit)
    Z = oracle.projection(X, R1, N, h, r)
    fb = check_tokens(Z, syn.bf16_bits_to_f64(R2), k, k + 6)
    assert fb < N  # the rule certifies most tokens


def test_window_holds_with_ties_and_near_ties():
    rng = np.random.default_rng(3)
    r, M, k = 16, 512, 8
    R2 = rng.integers(-2, 3, size=(r, M)).astype(np.float64)  # integer columns: many equal logits
    Z = rng.integers(-3, 4, size=(200, r)).astype(np.float64)
    check_tokens(Z, R2, k, k + 6)
    # near ties: two experts' columns differ by one bf16 step in one coordinate
    R2b = syn.bf16_bits_to_f64(syn.normal_bf16(0, 2, r, M, 0.25))
    for e in range(0, M, 37):
        R2b[:, e + 1 if e + 1 < M else e] = R2b[:, e]
        R2b[0, e] = bf16_round(np.array([R2b[0, e] * (1 + 2.0 ** -7)]))[0]
    Z = rng.standard_normal((200, r))
    check_tokens(Z, R2b, k, k + 6)
