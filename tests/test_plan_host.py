"""Host-side checks of the launch planner (spense_plan_shapes, no GPU): for
the workloads' shapes and token counts from 1 to 65535, every plan streams
every weight block exactly once (in pair mode once per CTA of a pair, whose
work tiles are pairs of 128-row tiles), keeps a cluster inside one tile, fits
the shared-memory and tensor-memory budgets of its CTAs-per-SM choice, covers
every token, and sizes its workspace for its partials; and the token-tile,
cluster and pair choices that the measurements justify are the ones made.
"""
import pytest

from dense_fp8_gemm_b200 import spense, workloads

SMS = 148
SMEM_MAX = 232448
RESERVE = 1024 + 2048  # alignment slack + barrier area

SHAPES = {
    "tiny": [(256, 512, 128)],
    "q": [(8192, 5120, 1280)],
    "k": [(1024, 5120, 1280)],
    "o": [(5120, 8192, 2048)],
    "qkv": [(8192, 5120, 1280), (1024, 5120, 1280), (1024, 5120, 1280)],
    "gateup": [(51200, 5120, 1280)],
    "down": [(5120, 25600, 6400)],
    "down_pure24": [(5120, 25600, 0)],
    "down_dense": [(5120, 25600, 25600)],
    "q36": [(10240, 5120, 1280)],
    "o36": [(5120, 10240, 2560)],
    "gateup36": [(55296, 5120, 1280)],
    "down36": [(5120, 27648, 6912)],
    "qkv36": [(10240, 5120, 1280), (1024, 5120, 1280), (1024, 5120, 1280)],
    "split": [(19200, 5120, 0), (6400, 5120, 5120)],           # output-split: 2:4 rows, dense rows
    "ragged": [(1000, 1024, 256), (136, 1024, 256)],
}
TOKENS = (1, 5, 8, 16, 32, 33, 64, 65, 128, 200, 256, 600, 4096, 65535)


def blocks_of(N, K, Kd):
    n_tiles = -(-N // 128)
    return n_tiles, -(-(K - Kd) // 256), -(-Kd // 128)


@pytest.mark.parametrize("name", sorted(SHAPES))
@pytest.mark.parametrize("M", TOKENS)
def test_plan_invariants(name, M):
    shapes = SHAPES[name]
    p = spense.plan_shapes(shapes, M, SMS)
    cps, S, grid, npad, pair = p["ctas_per_sm"], p["cluster"], p["grid"], p["npad"], p["pair"]
    # pair mode (CTA pairs, 256-row MMAs) is opt-in: never chosen by default
    assert pair == 0
    # tokens: tiles of npad (a multiple of 16) cover M, the last one not empty
    assert npad % 16 == 0 and 16 <= npad <= 256
    assert p["m_tiles"] * npad >= M > (p["m_tiles"] - 1) * npad
    # activation boxes: the valid rows of a tile, or each CTA's half of it in pair mode
    assert p["box_rows"] == (npad // 2 if pair else min(M, npad))
    # blocks: member by member, work tile by work tile (a 128-row tile, or a pair of them), every
    # token tile of a work tile
    total, tile_first = 0, []
    n_tiles = 0
    for N, K, Kd in shapes:
        nt, nsb, ndb = blocks_of(N, K, Kd)
        nt = -(-nt // 2) if pair else nt
        n_tiles += nt
        for _ in range(nt * p["m_tiles"]):
            tile_first.append(total)
            total += nsb + ndb
    tile_first.append(total)
    assert p["n_tiles"] == n_tiles and p["tiles"] == n_tiles * p["m_tiles"]
    assert p["total_blocks"] == total
    cs = p["cta_start"]
    assert cs[0] == 0 and cs[-1] == total and len(cs) == grid + 1
    assert all(a < b for a, b in zip(cs, cs[1:])), "a CTA with an empty or negative block range"
    # grid (work units: CTAs, or CTA pairs on two SMs each) and CTAs per SM
    assert cps in (1, 2) and 1 <= grid <= min(spense.PLAN_MAX_GRID, SMS * cps // (2 if pair else 1))
    if pair:
        assert cps == 1 and S == 1
    # cluster split: S consecutive CTAs share exactly one tile's blocks
    assert S in (1, 2, 4, 8)
    if S > 1:
        assert grid == p["tiles"] * S
        for t in range(p["tiles"]):
            assert cs[t * S] == tile_first[t] and cs[(t + 1) * S] == tile_first[t + 1]
        assert p["recv_bytes"] == (S - 1) * 128 * npad * 4
    else:
        assert p["recv_bytes"] == 0
    # shared memory: the ring (at least two stages) plus the receive area within the CTA's share
    any_sparse = any(K - Kd > 0 for _, K, Kd in shapes)
    xrows = npad // 2 if pair else npad  # token rows of a stage's activation tile in this CTA
    assert p["stage_bytes"] == 16384 + xrows * (256 if any_sparse else 128) + (4096 if any_sparse else 0)
    assert p["stages"] >= 2
    assert p["smem_bytes"] == RESERVE + p["stages"] * p["stage_bytes"] + p["recv_bytes"] + p["y_stage_bytes"]
    # whole-tile output staging (1 KB per epilogue warp) only for stream-K, and only where the ring leaves room
    assert p["y_stage_bytes"] in (0, 4096) and (S == 1 or p["y_stage_bytes"] == 0)
    assert p["smem_bytes"] <= SMEM_MAX // cps - (1024 if cps > 1 else 0)
    # tensor memory: a power of two from 32 columns holding the accumulators and the metadata
    assert p["tmem_cols"] in (32, 64, 128, 256, 512)
    assert p["nacc"] * npad + 16 <= p["tmem_cols"] <= 512 // cps
    # stream-K: the workspace holds every CTA's two fp32 partial slots (a cluster reduces in shared memory)
    if S == 1:
        assert p["workspace_bytes"] >= grid * (2 if pair else 1) * 2 * npad * 128 * 4
    assert p["l2_prefetch"] == (4 if S > 1 else 0)


@pytest.mark.parametrize("name,M,npad,S,cps,pair", [
    ("qkv", 16, 16, 2, 2, 0),      # the decode bench launch: clusters of 2, two CTAs per SM
    ("o", 16, 16, 4, 2, 0),        # o_proj: clusters of 4
    ("q", 64, 64, 2, 1, 0),
    ("q", 128, 64, 2, 2, 0),       # 128 tiles of 64 tokens: clusters only with two CTAs per SM
    ("gateup", 16, 16, 1, 1, 0),   # 400 row tiles: stream-K, one CTA per SM with a deep ring
    ("gateup", 128, 128, 1, 1, 0), # many tiles: token tiles of 128
    ("down", 256, 128, 1, 1, 0),   # a 94 MB weight with 160 tiles of 64: tiles of 128
    ("q", 256, 64, 1, 1, 0),       # a 30 MB weight: its repeated reads stay in L2, tiles of 64
    ("down36", 128, 128, 1, 1, 0), # 135 blocks per tile: no cluster split fits, so one token tile, not two of 64
    ("o36", 128, 128, 1, 1, 0),    # the same for o_proj (its tiles of 64 would be split over no cluster either)
    ("o36", 16, 16, 4, 2, 0),      # three stages at two CTAs per SM: clusters of 4 stay
    ("qkv36", 256, 96, 1, 1, 0),   # 128-token tiles: 1.3 per SM; 96: about 2 (45 MB stays in L2)
    ("down36", 600, 128, 1, 1, 0), # 102 MB: its re-reads would leave L2, tiles of 128 stay
    ("down36", 32, 32, 1, 1, 0),   # 40 tiles of 135 blocks: stream-K over every SM, not clusters of 2 on 80
    ("down36", 64, 64, 1, 1, 0),
    ("o36", 64, 64, 2, 1, 0),      # 50 blocks per tile: clusters of 2 stay
])
def test_plan_choices(name, M, npad, S, cps, pair):
    p = spense.plan_shapes(SHAPES[name], M, SMS)
    assert (p["npad"], p["cluster"], p["ctas_per_sm"], p["pair"]) == (npad, S, cps, pair)


def test_plan_workspace_layout():
    # status header (256 B), one arrival counter per tile (256-byte rounded), and for stream-K two fp32
    # partial slots of 128 rows x npad tokens per CTA (none for a cluster split, which reduces in shared
    # memory); no gather buffer for a tail dense region
    seen = set()
    for name in ("qkv", "gateup", "down", "split"):
        for M in (1, 16, 256, 600):
            p = spense.plan_shapes(SHAPES[name], M, SMS)
            ctas = 2 if p["pair"] else 1  # CTAs per work unit
            counters = -(-p["tiles"] * ctas * 4 // 256) * 256
            partials = 0 if p["cluster"] > 1 else p["grid"] * ctas * 2 * p["npad"] * 128 * 4
            assert p["workspace_bytes"] == 256 + counters + partials
            seen.add(p["cluster"] > 1)
    assert seen == {True, False}


def test_noalloc_scratch_fits_the_decoder_shapes_up_to_32_tokens():
    """spense_gemm_noalloc's fixed scratch holds the workspace of every 32B- and
    36B-class decoder weight (tail dense set) for M <= 32 on a 148-SM B200, as
    its header states."""
    for wl in (workloads.ATTN32B, workloads.FFN32B, workloads.CHAIN36B):
        for _, N, K in wl.shapes:
            for M in range(1, 33):
                p = spense.plan_shapes([(N, K, workloads.dense_count(K, 0.25))], M, SMS)
                assert p["workspace_bytes"] <= spense.NOALLOC_SCRATCH_BYTES, (wl.name, N, K, M)


def test_plan_rejects_bad_shapes():
    with pytest.raises(spense.SpenseError):
        spense.plan_shapes([(128, 520, 0)], 16)          # K not a multiple of 16
    with pytest.raises(spense.SpenseError):
        spense.plan_shapes([(128, 512, 0)], 0)           # no tokens
    with pytest.raises(spense.SpenseError):
        spense.plan_shapes([(128, 512, 0), (128, 1024, 0)], 16)  # members must share K
    with pytest.raises(spense.SpenseError):
        spense.plan_shapes([(128, 512, 0)] * 5, 16)      # at most four members
