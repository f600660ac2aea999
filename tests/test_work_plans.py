"""Host-side work plans of the tensor-core kernels (no device is touched).

The tcgen05 prefill attention cuts the items of its last, partial wave of SMs
into key ranges; the tcgen05 GEMM picks its token tile by how full the last
wave of tiles is.  The attention's plan decides how many partial-result slots
and item counters the kernel writes, so its invariants are memory safety:
every range holds at least one key tile, the ranges fit the scratch's slots
and the cut items its counters.  The exact plans of the 32768-token prompt's
chunks and the tile widths of the model's linears are the ones the GPU tests
and the bench ran.
"""
import itertools

import pytest

import qwen2_decode_step_b200 as q2


def item_tiles(rows, pos0, qt):
    """Key tiles of 128 that row block qt of a chunk at positions pos0.. sees
    (causal: up to the position of its last row)."""
    last = min(qt * 128 + 128, rows) - 1
    return (pos0 + last) // 128 + 1


@pytest.mark.parametrize("sms", [1, 2, 3, 7, 148])
def test_attention_plan_invariants(sms):
    for rows, pos0, nh in itertools.product([16, 100, 128, 129, 512, 1000, 4096],
                                            [0, 5, 128, 4096, 28672], [1, 2, 12, 14]):
        p = q2.q2_test_attn_plan(rows, pos0, nh, sms)
        ntq = (rows + 127) // 128
        items = ntq * nh
        assert p["items"] == items
        tail = items - p["n_whole"]
        if p["ts"] == 1:
            assert tail == 0 and p["ctas"] == items, (rows, pos0, nh, p)
            continue
        assert 2 <= p["ts"] <= 6, p
        # whole waves run whole; only the last, partial wave is cut
        assert tail == items % sms and 0 < tail < sms, (rows, pos0, nh, p)
        assert p["ctas"] == p["n_whole"] + tail * p["ts"]
        assert tail * p["ts"] <= p["slot_capacity"] and tail <= p["counter_capacity"], p
        # item i is row block ntq - 1 - i % ntq of head i // ntq: every range
        # of every cut item holds at least one key tile
        for i in range(p["n_whole"], items):
            assert item_tiles(rows, pos0, ntq - 1 - i % ntq) >= p["ts"], (rows, pos0, nh, i, p)


def test_attention_plan_of_the_32768_token_prompt():
    # eight chunks of 4096 rows, 12 query heads: 384 items of 128 rows on 148 SMs
    ts = [q2.q2_test_attn_plan(4096, 4096 * c, 12, 148)["ts"] for c in range(8)]
    assert ts == [1, 3, 5, 5, 5, 5, 5, 5]
    p = q2.q2_test_attn_plan(4096, 28672, 12, 148)
    assert (p["n_whole"], p["ctas"]) == (296, 296 + 88 * 5)


def test_attention_plan_with_one_tile_items_runs_whole():
    # a 512-token prompt: its first row block sees one key tile, so no item is cut
    p = q2.q2_test_attn_plan(512, 0, 12, 148)
    assert p["ts"] == 1 and p["ctas"] == 48


@pytest.mark.parametrize("args", [(0, 0, 12, 148), (512, 0, 0, 148), (512, 0, 12, 0), (1 << 30, 0, 12, 148)])
def test_attention_plan_rejects_bad_arguments(args):
    with pytest.raises(q2.Q2Error):
        q2.q2_test_attn_plan(*args)


@pytest.mark.parametrize("M,N,bn", [
    (64, 2048, 64), (100, 1536, 64), (128, 1536, 128), (255, 17920, 128),
    # the 4096-token prefill chunk: q/k/v 256 tiles of 256 fill two waves; o and
    # down take 192 (264 tiles in two waves, where 192 tiles of 256 leave the
    # second a third full); gate/up stays at 256
    (4096, 2048, 256), (4096, 1536, 192), (4096, 17920, 256),
    (32768, 2048, 256), (32768, 1536, 256), (32768, 17920, 256),
    (512, 2048, 192), (512, 1536, 192), (512, 17920, 256), (300, 1000, 192), (257, 640, 192),
])
def test_gemm_token_tile(M, N, bn):
    assert q2.q2_test_gemm_tile(M, N, 148) == bn
