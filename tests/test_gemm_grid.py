"""Host checks of the active-row GEMM's launch rule and work split (no GPU).

`gemm_launch` picks an activation-tile width, k-blocks per ring stage and a
grid (whole tiles, equal k pieces of a tile, or the stream-K share), and the
kernel gives CTA c the (tile, k-block) items [T*c/G, T*(c+1)/G).  A tile split
over several CTAs is summed through the partial buffer (two slots per CTA: its
first and its last tile) and one arrival counter per tile, unless its pieces
add straight into the residual stream.  These tests restate the rule as the
source writes it and check, for every GEMM of every workload shape over a
sweep of row counts and SM counts, what the kernel relies on:

* every item belongs to exactly one CTA;
* a split tile is only ever the first or the last tile of a CTA's range, its
  partial slot lies inside the buffer the workspace sizing provides, and its
  counter index inside the counter array;
* the owner range the last-piece logic computes from the closed form equals
  the CTAs that really hold pieces of the tile, each exactly once.
"""
import pytest

K_BK = 64
EPI_STORE_F32, EPI_RESID_ADD, EPI_SWIGLU, EPI_LMHEAD = "f32", "resid", "swiglu", "lmhead"

SHAPES = {  # name: (d, qkvd, qd, F, V)
    "tiny": (256, 768, 256, 1024, 1024),
    "parity": (512, 1024, 512, 1408, 4096),
    "llada8b": (4096, 12288, 4096, 12288, 126464),
    "dream7b": (3584, 4608, 3584, 18944, 152064),
}
ROWS = sorted({1, 7, 16, 17, 32, 33, 63, 64, 65, 100, 128, 129, 160, 205, 256, 257, 300, 384, 385, 400, 512,
               513, 600, 640, 700, 768, 769, 1024, 1536, 2048, 3072, 4096, 5120, 8448, 12288})


def pick_bn(rows):
    if rows <= 16:
        return 16
    if rows <= 32:
        return 32
    if rows <= 64:
        return 64
    return 128 if rows <= 512 else 256


def max_ksub(bn):
    return 4 if bn <= 64 else (2 if bn <= 128 else 1)


def pick_ksub(K, bn):
    want = min(4, max_ksub(bn))
    for k in (4, 2, 1):
        if k <= want and (K // K_BK) % k == 0:
            return k
    return 1


def whole_piece_grid(tiles, KB, sms, max_whole_per_cta=4):
    if tiles >= sms:
        per = -(-tiles // sms)
        if per > max_whole_per_cta and 4 * (per * sms - tiles) >= sms:
            return 0
        return -(-tiles // per)
    p = max(1, min(sms // tiles, KB // 32))
    while p > 1 and KB % p:
        p -= 1
    return tiles * p


def launch(rows, n_tiles_w, K, kind, sms, partial_floats, n_counters, wide_ok=False):
    """The launch shape gemm_launch chooses: (bn, tiles, KB, grid, add_pieces)."""
    bn = pick_bn(rows)
    if wide_ok and bn == 128 and 128 < rows <= 256:
        bn = 256
    if kind == EPI_SWIGLU and bn == 128 and rows > 384:
        bn = 256
    if kind == EPI_RESID_ADD and bn == 128 and n_tiles_w * -(-rows // 128) > sms:
        bn = 256
    tiles = n_tiles_w * -(-rows // bn)
    KB = K // (K_BK * pick_ksub(K, bn))
    grid = min(sms, tiles * KB)
    add_pieces = kind == EPI_RESID_ADD and bn >= 128 and 2 * tiles <= sms
    if bn >= 128 and not add_pieces:
        wg = whole_piece_grid(tiles, KB, sms)
        if wg > 0:
            grid = wg
    grid = min(grid, tiles * KB)
    need = grid * 2 * bn * 128
    if not add_pieces and (partial_floats < need or n_counters < tiles):
        if (tiles * KB) % grid != 0 or tiles % grid != 0:
            grid = min(grid, tiles)
        while grid > 1 and tiles % grid != 0:
            grid -= 1
    return bn, tiles, KB, grid, add_pieces


def sk_lo(T, G, c):
    return T * c // G


def sk_first_cta(x, T, G):
    return ((x + 1) * G + T - 1) // T - 1


def check_split(bn, tiles, KB, grid, add_pieces, partial_floats, n_counters):
    T = tiles * KB
    owners = [[] for _ in range(tiles)]
    covered = 0
    for c in range(grid):
        lo, hi = sk_lo(T, grid, c), sk_lo(T, grid, c + 1)
        assert lo == covered and hi > lo                 # contiguous, non-empty, in CTA order
        covered = hi
        first, last = lo // KB, (hi - 1) // KB
        for tile in range(first, last + 1):
            owners[tile].append(c)
    assert covered == T
    for tile, cs in enumerate(owners):
        whole = len(cs) == 1
        if whole or add_pieces:
            continue
        assert tile < n_counters
        x0 = tile * KB
        assert (sk_first_cta(x0, T, grid), sk_first_cta(x0 + KB - 1, T, grid)) == (cs[0], cs[-1])
        assert cs == list(range(cs[0], cs[-1] + 1))
        for c in cs:
            lo, hi = sk_lo(T, grid, c), sk_lo(T, grid, c + 1)
            which = 0 if tile == lo // KB else 1
            assert which == 0 or tile == (hi - 1) // KB   # only a range's first or last tile is split
            assert (c * 2 + which + 1) * bn * 128 <= partial_floats


def gemms(d, qkvd, qd, F, V):
    """(name, n_tiles_w, K, epilogue kind, wide_ok) of the layer GEMMs and the vocabulary projection."""
    return [("qkv", qkvd // 128, d, EPI_STORE_F32, True), ("o", d // 128, qd, EPI_RESID_ADD, False),
            ("gate_up", F // 64, d, EPI_SWIGLU, False), ("down", d // 128, F, EPI_RESID_ADD, False),
            ("lm_head", V // 128, d, EPI_LMHEAD, False)]


@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("sms", [148, 132, 100])
def test_engine_gemm_splits_fit_the_workspace(shape, sms):
    """Engine sizing: partial floats = SMs x 2 x pick_bn(rows) x 128, one counter per
    pick_bn-wide tile (the launch only ever widens the tile, so tiles never outnumber them)."""
    for name, n_tiles_w, K, kind, wide_ok in gemms(*SHAPES[shape]):
        for rows in ROWS:
            pf = sms * 2 * pick_bn(rows) * 128
            nc = n_tiles_w * -(-rows // pick_bn(rows))
            bn, tiles, KB, grid, add_pieces = launch(rows, n_tiles_w, K, kind, sms, pf, nc, wide_ok)
            assert tiles <= nc, (name, rows)
            assert 1 <= grid <= sms
            check_split(bn, tiles, KB, grid, add_pieces, pf, nc)


@pytest.mark.parametrize("shape", list(SHAPES))
def test_op_gemm_scratch_falls_back_to_whole_tiles(shape):
    """The single-GEMM op counts its counters with 128-wide tiles up to 128 rows and 256-wide
    above: where the launch's tiles outnumber them, the grid divides the tiles and no tile
    is split."""
    sms = 148
    for name, n_tiles_w, K, kind, wide_ok in gemms(*SHAPES[shape]):
        for rows in ROWS:
            b = 16 if rows <= 16 else 32 if rows <= 32 else 64 if rows <= 64 else 128 if rows <= 128 else 256
            nc = n_tiles_w * -(-rows // b)
            pf = sms * 2 * pick_bn(rows) * 128
            bn, tiles, KB, grid, add_pieces = launch(rows, n_tiles_w, K, kind, sms, pf, nc, wide_ok)
            if tiles > nc and not add_pieces:
                assert tiles % grid == 0, (name, rows)
            check_split(bn, tiles, KB, grid, add_pieces, pf, nc)


def test_tile_width_rule():
    """The measured widths: 128 up to 512 rows, 256 above; QKV (caller opt-in) at 129-256 rows,
    gate/up from 385 rows and the residual GEMMs where 128-wide tiles outnumber the SMs."""
    d, qkvd, qd, F, V = SHAPES["llada8b"]
    big = 10 ** 12
    width = lambda rows, *g: launch(rows, *g, sms=148, partial_floats=big, n_counters=big)[0]
    assert [width(r, qkvd // 128, d, EPI_STORE_F32) for r in (64, 65, 512, 513)] == [64, 128, 128, 256]
    assert [launch(r, qkvd // 128, d, EPI_STORE_F32, 148, big, big, wide_ok=True)[0]
            for r in (128, 129, 256, 257)] == [128, 256, 256, 128]
    assert [width(r, F // 64, d, EPI_SWIGLU) for r in (384, 385, 512)] == [128, 256, 256]
    assert [width(r, d // 128, F, EPI_RESID_ADD) for r in (512, 513)] == [128, 256]
    assert width(384, 64, 8192, EPI_RESID_ADD) == 256          # 64 x 3 = 192 tiles > 148 SMs


def test_restated_rule_matches_the_source():
    """The thresholds restated above are the ones gemm_tc.cu uses (a change there must be
    carried here, or these checks would test a stale rule)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "token_skip_denoising_b200", "csrc",
                            "gemm_tc.cu")).read()
    assert re.search(r"if \(rows <= 512\) return 128;\s*return 256;", src)
    assert "a.wide_ok && bn == 128 && a.rows_cap > 128 && a.rows_cap <= 256) bn = 256;" in src
    assert "a.swiglu && bn == 128 && a.rows_cap > 384) bn = 256;" in src
    assert "a.epi.kind == EPI_RESID_ADD && bn == 128 &&" in src
    assert "a.epi.kind == EPI_RESID_ADD && bn >= 128 && 2 * tiles <= num_sms();" in src
    assert "constexpr int kMaxWholePerCta = 4;" in src
    assert "per > kMaxWholePerCta && 4 * (static_cast<int64_t>(per) * sms - tiles) >= sms" in src
    assert "std::max(1, std::min(sms / tiles, KB / 32));" in src
    assert "constexpr int max_ksub(int bn) { return bn <= 64 ? 4 : (bn <= 128 ? 2 : 1); }" in src
    dev = open(os.path.join(os.path.dirname(__file__), "..", "token_skip_denoising_b200", "csrc",
                            "gemm_dev.cuh")).read()
    assert "return T * c / G;" in dev and "((x + 1) * G + T - 1) / T - 1" in dev
