"""Planted mistakes: copies of the oracle with one plausible bug each must fail
at least one pin.  This shows the pins can tell a right oracle from a wrong one.
(All on the CPU; nothing here touches a GPU.)"""
import types

import numpy as np
import pytest

import oracle
from tests import oracle_pins

ORDER_OK = (0, 2, 4, 6, 1, 3, 5, 7)


def make_impl(sign_flip=False, reverse_stages=False, swap_roles=False, no_scale=False,
              theta_global=False, order=ORDER_OK, no_zero=False, group0_scale=False,
              inverse_forward_order=False, shared_group_base=False, q_half_away=False,
              q_clamp7=False, q_no_offset=False, w_scale_multiplied=False, q_group0_scale=False,
              q_no_bound=False, w_no_stages=False, qw_no_stages=False, qw_untransposed=False,
              moe_bias0=False, moe_wrap_invalid=False, moe_no_rotation=False, moe_slot_transposed=False):
    def stage_idx(pairs_s, G):
        K = pairs_s.shape[0]
        local = pairs_s.astype(np.int64)
        base = 0 if shared_group_base else (np.arange(K // 2) // (G // 2)) * G
        i, j = local[0::2] + base, local[1::2] + base
        return (j, i) if swap_roles else (i, j)

    def apply_stage(X, pairs_s, theta_s, G, sgn=1.0):
        i, j = stage_idx(pairs_s, G)
        t = sgn * np.asarray(theta_s, np.float64)
        if theta_global:
            t = t[::-1]
        c, s = np.cos(t), np.sin(t)
        a, b = X[:, i].copy(), X[:, j].copy()
        X[:, i] = a * c + b * s
        X[:, j] = (a * s if sign_flip else -a * s) + b * c

    def rotate(x, cs, pairs, theta, group_size, krot=None):
        X = np.array(x, np.float64)
        G = oracle.normalize_group_size(group_size, X.shape[1])
        if cs is not None and not no_scale:
            X *= np.asarray(cs, np.float64)
        if krot is None:
            krot = 0 if pairs is None else pairs.shape[0]
        order = reversed(range(krot)) if reverse_stages else range(krot)
        for s in order:
            apply_stage(X, pairs[s], theta[s], G)
        return X

    def inverse_rotate(xr, cs, pairs, theta, group_size):
        X = np.array(xr, np.float64)
        G = oracle.normalize_group_size(group_size, X.shape[1])
        order = range(pairs.shape[0]) if inverse_forward_order else reversed(range(pairs.shape[0]))
        for s in order:
            apply_stage(X, pairs[s], theta[s], G, sgn=-1.0)
        if cs is not None and not no_scale:
            X /= np.asarray(cs, np.float64)
        return X

    def awq_pack(codes, zeros, G):
        N = codes.shape[0]

        def pk(c):
            w = np.zeros((c.shape[1], N // 8), np.uint64)
            for t in range(8):
                w |= c.T.astype(np.uint64)[:, order[t]::8] << np.uint64(4 * t)
            return w.astype(np.uint32).view(np.int32)
        return pk(codes), pk(zeros)

    def awq_unpack(qw, qz, N, K, G):
        def up(words):
            w = np.asarray(words).view(np.uint32).astype(np.uint64)
            out = np.zeros((w.shape[0], N), np.uint8)
            for t in range(8):
                out[:, order[t]::8] = ((w >> np.uint64(4 * t)) & np.uint64(15)).astype(np.uint8)
            return out.T.copy()
        return up(qw), up(qz)

    def dequant(codes, zeros, scales, G):
        q = codes.T.astype(np.float64)
        z = np.repeat(zeros.T.astype(np.float64), G, axis=0)
        s = np.repeat(np.asarray(scales, np.float64), G, axis=0)
        if group0_scale:
            s = np.repeat(np.asarray(scales, np.float64)[:1], q.shape[0], axis=0)
        return (q if no_zero else q - z) * s

    def w4_linear_from_codes(x, codes, zeros, scales, bias, cs, pairs, theta, G, krot):
        Y = rotate(x, cs, pairs, theta, G, krot=krot) @ dequant(codes, zeros, scales, G)
        if bias is not None:
            Y += np.asarray(bias, np.float64)
        return Y

    def transform_weight(W, cs, pairs, theta, group_size, krot=None):
        D = None if cs is None else (np.asarray(cs, np.float64) if w_scale_multiplied
                                     else 1.0 / np.asarray(cs, np.float64))
        if w_no_stages:
            krot = 0
        return rotate(W, D, pairs, theta, group_size, krot=krot)

    def quantize_sym4(W_r, scales, G):
        W_r = np.asarray(W_r, np.float64)
        N, K = W_r.shape
        sc = np.asarray(scales, np.float64)
        if not q_no_bound:
            sc = np.clip(sc, 1e-5, 1e5)
        if q_group0_scale:
            sc = np.repeat(sc[:1], sc.shape[0], axis=0)
        with np.errstate(divide="ignore", invalid="ignore"):
            t = W_r / np.repeat(sc.T, G, axis=1)
        q = np.sign(t) * np.floor(np.abs(t) + 0.5) if q_half_away else np.rint(t)
        q = np.nan_to_num(q, nan=0.0, posinf=99.0, neginf=-99.0)
        q = np.clip(q, -7 if q_clamp7 else -8, 7)
        codes = (q.astype(np.int64) & 15).astype(np.uint8) if q_no_offset else (q + 8).astype(np.uint8)
        return codes, np.full((N, K // G), 0 if q_no_offset else 8, np.uint8)

    def quantize_weight(W, cs, pairs, theta, scales, G, krot=None):
        W_r = transform_weight(W, cs, pairs, theta, G, krot=0 if qw_no_stages else krot)
        codes, zeros = quantize_sym4(W_r, scales, G)
        if qw_untransposed:                   # words built along the wrong axis
            return awq_pack(np.ascontiguousarray(codes.reshape(codes.shape[1], codes.shape[0])), zeros, G)
        return awq_pack(codes, zeros, G)

    def moe_linear_from_codes(x, idx, codes, zeros, scales, bias, cs, pairs, theta, G, krot):
        idx = np.asarray(idx).astype(np.int64)
        T, topk = idx.shape
        E, N = codes.shape[0], codes.shape[1]
        xr = np.array(x, np.float64) if moe_no_rotation else rotate(x, cs, pairs, theta, G, krot=krot)
        y = np.zeros((T, topk, N))
        for t in range(T):
            for j in range(topk):
                e = int(idx[j % T, t % topk]) if moe_slot_transposed else int(idx[t, j])
                if moe_wrap_invalid:
                    e %= E                         # an index past the experts wraps around
                elif not 0 <= e < E:
                    continue
                y[t, j] = xr[t] @ dequant(codes[e], zeros[e], scales[e], G)
                if bias is not None:
                    y[t, j] += np.asarray(bias[0 if moe_bias0 else e], np.float64)
        return y

    return types.SimpleNamespace(rotate=rotate, inverse_rotate=inverse_rotate, awq_pack=awq_pack,
                                 awq_unpack=awq_unpack, dequant=dequant,
                                 w4_linear_from_codes=w4_linear_from_codes,
                                 transform_weight=transform_weight, quantize_sym4=quantize_sym4,
                                 quantize_weight=quantize_weight, moe_linear_from_codes=moe_linear_from_codes)


def failing_pins(impl):
    bad = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(impl)
        except (AssertionError, IndexError, ValueError):
            bad.append(pin.__name__)
    return bad


def test_unmutated_copy_passes_all_pins():
    assert failing_pins(make_impl()) == []


MUTATIONS = {
    "sign_flip": dict(sign_flip=True),
    "reverse_stages": dict(reverse_stages=True),
    "swap_pair_roles": dict(swap_roles=True),
    "dropped_channel_scale": dict(no_scale=True),
    "theta_misindexed": dict(theta_global=True),
    "identity_nibble_order": dict(order=tuple(range(8))),
    "dropped_zero_point": dict(no_zero=True),
    "scale_group_misindexed": dict(group0_scale=True),
    "inverse_not_reversed": dict(inverse_forward_order=True),
    "pairs_not_group_local": dict(shared_group_base=True),
    "quant_ties_away_from_zero": dict(q_half_away=True),
    "quant_clamped_to_plus_minus_7": dict(q_clamp7=True),
    "quant_twos_complement_codes": dict(q_no_offset=True),
    "weight_scaled_by_cs_not_its_inverse": dict(w_scale_multiplied=True),
    "quant_scale_group_misindexed": dict(q_group0_scale=True),
    "quant_scale_unbounded": dict(q_no_bound=True),
    "weight_stages_skipped": dict(w_no_stages=True),
    "quantize_weight_drops_the_stages": dict(qw_no_stages=True),
    "quantize_weight_packs_untransposed_codes": dict(qw_untransposed=True),
    "moe_bias_of_the_first_expert": dict(moe_bias0=True),
    "moe_invalid_index_wraps_around": dict(moe_wrap_invalid=True),
    "moe_rotation_skipped": dict(moe_no_rotation=True),
    "moe_slots_read_transposed": dict(moe_slot_transposed=True),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_is_caught(name):
    assert failing_pins(make_impl(**MUTATIONS[name])), name
