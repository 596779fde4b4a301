"""Pins of the paged-cache oracle (oracle.attn_paged, oracle.paged_append):
the same logical cache in blocks gives exactly the packed-cache oracle's
result, whatever the physical order of the blocks, and appending the new
tokens' rows gives the result of having them in the cache already."""
import numpy as np
import pytest

import oracle
from io_aware_exact_29_b200.workloads import DecodeCase, kvcache_inputs, paged_from_packed


@pytest.mark.parametrize("block_size", [1, 3, 16, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_paged_equals_packed(block_size, causal):
    c = DecodeCase("p", 4, 8, 2, 3, 16, (1, 90), causal, slack=4)
    inp = kvcache_inputs(c, seed=11, seqlens=[90, 1, 0, 37])
    pg = paged_from_packed(inp, block_size, seed=11)
    o_ref, l_ref = oracle.attn_kvcache(inp["q"], inp["k_cache"], inp["v_cache"],
                                       inp["cu_seqlens_k"], inp["seqlens_k"], c.scale, causal)
    o, lse = oracle.attn_paged(inp["q"], pg["k_cache"], pg["v_cache"], pg["block_table"],
                               pg["seqlens_k"], c.scale, causal)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, l_ref)


def test_block_order_does_not_matter():
    c = DecodeCase("p", 3, 4, 1, 2, 8, (1, 50), True)
    inp = kvcache_inputs(c, seed=12, seqlens=[50, 20, 33])
    a = oracle.attn_paged(inp["q"], **{k: v for k, v in paged_from_packed(inp, 8, seed=1).items()
                                       if k != "seqlens_k"}, seqlens_k=inp["seqlens_k"],
                          scale=c.scale, causal=True)
    b = oracle.attn_paged(inp["q"], **{k: v for k, v in paged_from_packed(inp, 8, seed=2).items()
                                       if k != "seqlens_k"}, seqlens_k=inp["seqlens_k"],
                          scale=c.scale, causal=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_append_writes_the_new_rows():
    c = DecodeCase("p", 3, 8, 2, 4, 16, (4, 70), True)
    inp = kvcache_inputs(c, seed=13, seqlens=[70, 4, 19])
    full = paged_from_packed(inp, 16, seed=13)
    holes = paged_from_packed(inp, 16, seed=13, new_tokens=4)
    # the holes are NaN until the append
    kc, vc = oracle.paged_append(holes["k_cache"], holes["v_cache"], holes["block_table"],
                                 holes["seqlens_k"], holes["k_new"], holes["v_new"])
    assert np.array_equal(kc, full["k_cache"].double().numpy(), equal_nan=True)
    assert np.array_equal(vc, full["v_cache"].double().numpy(), equal_nan=True)
    o1, l1 = oracle.attn_paged(inp["q"], full["k_cache"], full["v_cache"], full["block_table"],
                               full["seqlens_k"], c.scale, True)
    o2, l2 = oracle.attn_paged(inp["q"], holes["k_cache"], holes["v_cache"],
                               holes["block_table"], holes["seqlens_k"], c.scale, True,
                               k_new=holes["k_new"], v_new=holes["v_new"])
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
