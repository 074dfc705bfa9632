"""Pins the oracle's paged prefill attention: causal attention of each sequence's
new tokens over its cached keys and values, against torch's fp64
scaled-dot-product attention with the causal (whole prompt) or position mask
(chunk on top of earlier context), plus the decode special case."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
import workloads
from oracle_side import raw, run_script


def _sdpa_rows(wl, b, qrows):
    """torch fp64 reference for sequence b: qrows [n_new, Hq, D] (fp64)."""
    seq = int(wl.batch[b])
    n = int(wl.context_lens()[b])
    m = int(wl.n_new[b])
    k = wl.contiguous_kv(seq, 0).double().permute(1, 0, 2).repeat_interleave(wl.G, 0)
    v = wl.contiguous_kv(seq, 1).double().permute(1, 0, 2).repeat_interleave(wl.G, 0)
    q = qrows.permute(1, 0, 2)                     # [Hq, m, D]
    pos = torch.arange(n - m, n)[:, None]
    mask = torch.arange(n)[None, :] <= pos         # [m, n]
    if m == n:
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=wl.scale)
    else:
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=wl.scale)
    return o.permute(1, 0, 2)                      # [m, Hq, D]


def _case(dtype, ctx, n_new, G=4, seed=3):
    return workloads.prefill("p", dtype, 4 * G, 4, 64, 16, ctx, n_new, seed)


def test_prefill_matches_library_attention_whole_prompts_and_chunks():
    wl = _case("f32", [1, 17, 64, 300, 90], [1, 17, 30, 120, 90])
    o = run_script(wl)
    qs = workloads.query_start(wl)
    q = workloads.q_prefill(wl)
    out = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], qs, wl.scale, wl.dtype)
    for b in range(wl.B):
        ref = _sdpa_rows(wl, b, q[qs[b]:qs[b + 1]].double())
        np.testing.assert_allclose(out[qs[b]:qs[b + 1]], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_prefill_of_16_bit_inputs_uses_their_exact_values():
    wl = _case("bf16", [40, 70], [40, 33], G=2, seed=4)
    o = run_script(wl)
    qs = workloads.query_start(wl)
    q = workloads.q_prefill(wl)
    out = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], qs, wl.scale, wl.dtype)
    for b in range(wl.B):
        ref = _sdpa_rows(wl, b, q[qs[b]:qs[b + 1]].double())
        np.testing.assert_allclose(out[qs[b]:qs[b + 1]], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_one_new_token_is_decode_and_rows_are_independent():
    wl = _case("f16", [5, 33, 200], [1, 1, 1], seed=6)
    o = run_script(wl)
    qs = workloads.query_start(wl)
    q = workloads.q_prefill(wl)
    out = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], qs, wl.scale, wl.dtype)
    dec = oracle.paged_decode_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                        o["ctx"], wl.scale, wl.dtype)
    assert np.array_equal(out, dec)
    rows = [1, 5, 2 * wl.Hq + 3]
    part = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                          o["ctx"], qs, wl.scale, wl.dtype, rows=rows)
    flat = part.reshape(-1, wl.D)
    assert np.array_equal(flat[rows], out.reshape(-1, wl.D)[rows])
    assert np.isnan(flat[0]).all()


def test_more_new_tokens_than_context_is_rejected():
    wl = _case("f32", [10], [10])
    o = run_script(wl)
    q = np.zeros((11, wl.Hq, wl.D), np.float32)
    try:
        oracle.paged_prefill_attention(q, o["k_cache"], o["v_cache"], o["table"], o["ctx"],
                                       [0, 11], wl.scale, wl.dtype)
    except ValueError:
        return
    raise AssertionError("accepted n_new > ctx")


def test_prefill_at_head_dim_128_with_groups_of_8():
    """The shapes the GPU parity cases run (head_dim 128, eight query heads per kv
    head): a chunk after context, a whole prompt and a single token, against torch."""
    wl = workloads.prefill("p128", "f16", 16, 2, 128, 16, [150, 37, 9], [20, 37, 1], 9)
    o = run_script(wl)
    qs = workloads.query_start(wl)
    q = workloads.q_prefill(wl)
    out = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], qs, wl.scale, wl.dtype)
    for b in range(wl.B):
        ref = _sdpa_rows(wl, b, q[qs[b]:qs[b + 1]].double())
        np.testing.assert_allclose(out[qs[b]:qs[b + 1]], ref.numpy(), rtol=1e-12, atol=1e-12)
