"""Host checks of the fused layer kernel's work partitions (no GPU).

The persistent kernel splits its work with a few integer formulas; an error
in one of them would drop or repeat work (or index out of bounds) only for
some shapes.  These tests restate each formula as the kernel source writes it
and check, over every shape the workloads and the parity tests use and a
sweep around them, the property the kernel relies on:

* the stream-K split of a GEMM's (tile, k-block) items gives every item to
  exactly one CTA, in contiguous ranges;
* the ES choice's column slices of a row cover [0, d) once, in 128-column
  chunks, for any number of slices;
* the attention key splits cover every 64-key block once and the query tiles
  every (row, head) unit once;
* the RoPE step's 4-pair items rotate every (low, high) pair of a row once,
  inside one head, with their vector loads and stores aligned;
* choosing the k candidates whose rank (higher score first, ties to the lower
  position) is below k picks the same set, in ascending positions, as the
  selection kernel's rule "the k highest scores, ties to the lower position"
  (stated here as a stable sort).
"""
import numpy as np
import pytest

K_BK, K_KSUB, N_SMS, KEYS_PER_BLOCK, UNITS_PER_CTA = 64, 2, 148, 64, 64

LAYER_SHAPES = [  # (d, qkvd, qd, F): tiny, the parity shapes, LLaDA-8B, Dream-7B
    (256, 768, 256, 1024), (512, 1024, 512, 1408), (1024, 1536, 1024, 2816),
    (4096, 12288, 4096, 12288), (3584, 4608, 3584, 18944),
]


def items_of(K, n_tiles, G, c):
    KB = K // (K_BK * K_KSUB)
    T = n_tiles * KB
    Gg = min(T, G)
    lo = T * c // Gg if c < Gg else 0
    hi = T * (c + 1) // Gg if c < Gg else 0
    return lo, hi, KB


@pytest.mark.parametrize("d,qkvd,qd,F", LAYER_SHAPES)
def test_stream_k_items_are_a_partition(d, qkvd, qd, F):
    gemms = [(d, qkvd // 128), (qd, d // 128), (d, 2 * F // 128), (F, d // 128)]
    for K, n_tiles in gemms:
        T = n_tiles * (K // (K_BK * K_KSUB))
        owner = np.full(T, -1)
        prev_hi = 0
        for c in range(N_SMS):
            lo, hi, KB = items_of(K, n_tiles, N_SMS, c)
            if hi > lo:
                assert lo == prev_hi                   # contiguous, in CTA order
                prev_hi = hi
            assert np.all(owner[lo:hi] == -1)
            owner[lo:hi] = c
        assert np.all(owner >= 0) and prev_hi == T


def slices(d, nrow, G=N_SMS):
    nch = d >> 7
    S = max(1, min(nch, (G * 4) // nrow))
    return [((nch * sl // S) << 7, min(d, (nch * (sl + 1) // S) << 7)) for sl in range(S)]


@pytest.mark.parametrize("d", [256, 512, 1024, 3584, 4096])
@pytest.mark.parametrize("nrow", [1, 7, 8, 16, 32, 37, 64, 100, 148, 592, 593, 2048, 32768])
def test_eq1_column_slices_cover_each_row_once(d, nrow):
    cover = np.zeros(d, int)
    for i0, i1 in slices(d, nrow):
        assert i0 % 128 == 0 and i1 % 128 == 0 and i0 < i1
        cover[i0:i1] += 1
    assert np.all(cover == 1)


def attn_geometry(B, Hq, Hkv, rows_per_seq, N, splits_env=0):
    Gq = Hq // Hkv
    units = rows_per_seq * Gq
    qtiles = (units + 63) // 64
    n_blocks = (N + 63) // 64
    groups = B * Hkv * qtiles
    splits = splits_env if splits_env > 0 else max(1, N_SMS // groups)
    splits = max(1, min(n_blocks, splits))
    bps = (n_blocks + splits - 1) // splits
    splits = (n_blocks + bps - 1) // bps
    return qtiles, n_blocks, splits, bps


@pytest.mark.parametrize("B,Hq,Hkv,rows,N", [
    (1, 32, 32, 7, 768), (1, 32, 32, 32, 768), (2, 4, 4, 8, 64), (2, 8, 2, 33, 130), (8, 28, 4, 9, 1536),
    (4, 32, 32, 64, 5120), (1, 4, 2, 1, 65), (3, 4, 2, 64, 130),
])
@pytest.mark.parametrize("splits_env", [0, 1, 3, 16])
def test_attention_splits_cover_keys_and_units(B, Hq, Hkv, rows, N, splits_env):
    qtiles, n_blocks, splits, bps = attn_geometry(B, Hq, Hkv, rows, N, splits_env)
    blocks = np.zeros(n_blocks, int)
    for s in range(splits):
        blk0, blk1 = s * bps, min(n_blocks, s * bps + bps)
        assert blk0 < blk1                             # no empty split after the rounding
        blocks[blk0:blk1] += 1
    assert np.all(blocks == 1)
    units = rows * (Hq // Hkv)
    cover = np.zeros(units, int)
    for qt in range(qtiles):
        u0 = qt * UNITS_PER_CTA
        cover[u0:min(units, u0 + UNITS_PER_CTA)] += 1
    assert np.all(cover == 1)


def order_key(x):
    """The kernels' monotone score key (NaN lowest, -0 == +0), as uint32."""
    x = np.float32(x)
    if np.isnan(x):
        return 0
    x = np.float32(x + np.float32(0.0))
    u = int(np.array([x], np.float32).view(np.uint32)[0])
    return (~u & 0xFFFFFFFF) if (u & 0x80000000) else (u | 0x80000000)


def rank_count_choice(scores, k):
    keys = [order_key(s) for s in scores]
    n = len(keys)
    chosen = [sum(1 for j in range(n) if keys[j] > keys[i] or (keys[j] == keys[i] and j < i)) < k
              for i in range(n)]
    return [i for i in range(n) if chosen[i]]


def stable_topk(scores, k):
    s = np.asarray(scores, np.float32)
    key = np.where(np.isnan(s), -np.inf, s)
    order = np.argsort(-key, kind="stable")           # ties keep the lower position first
    return sorted(order[:k].tolist())


@pytest.mark.parametrize("seed", range(40))
def test_rank_count_choice_is_the_selection_rule(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 70))
    k = int(rng.integers(1, n + 1))
    kind = seed % 4
    if kind == 0:
        s = rng.standard_normal(n)
    elif kind == 1:
        s = rng.integers(0, 3, n).astype(float)        # many ties
    elif kind == 2:
        s = rng.choice([0.0, -0.0, 1.0, -1.0], n)      # signed zeros tie
    else:
        s = rng.standard_normal(n)
        s[rng.random(n) < 0.3] = np.nan                # NaN ranks lowest
    got = rank_count_choice(s, k)
    assert len(got) == k
    if kind == 3:
        # NaN candidates are chosen only once every number is (lowest positions first)
        num = [i for i in range(n) if not np.isnan(s[i])]
        want = stable_topk(s, k) if k <= len(num) else sorted(
            num + [i for i in range(n) if np.isnan(s[i])][:k - len(num)])
        assert got == want
    else:
        assert got == stable_topk(s, k)


def rope_items(qkvd, hd):
    """The fused kernel's RoPE items of one row: item rr covers pairs pi..pi+3 of head rr / (hd/8),
    element nlo (low half) and nlo + hd/2 (high half) of the row's QKV sums."""
    half, groups, gph = hd // 2, qkvd >> 3, (hd // 2) >> 2
    out = []
    for rr in range(groups):
        head = rr // gph
        pi = (rr - head * gph) * 4
        out.append((head * hd + pi, pi))
    return out, half


@pytest.mark.parametrize("Hq,Hkv,hd", [(4, 4, 64), (8, 2, 128), (28, 4, 128), (32, 32, 128), (4, 2, 64)])
def test_rope_items_cover_each_pair_once_aligned(Hq, Hkv, hd):
    """Every (low, high) element pair of a row is rotated exactly once; a 4-pair item never
    crosses a head, and its 16-byte loads (fp32 sums, cos/sin rows) and 8-byte stores (bf16 q and
    cache rows) start on their alignment for every row and position."""
    qd, kvd = Hq * hd, Hkv * hd
    qkvd = qd + 2 * kvd
    items, half = rope_items(qkvd, hd)
    seen = np.zeros(qkvd, dtype=int)
    for nlo, pi in items:
        assert nlo % 4 == 0 and pi % 4 == 0 and pi + 3 < half
        assert nlo // hd == (nlo + half + 3) // hd          # both halves in one head
        for k in range(4):
            seen[nlo + k] += 1
            seen[nlo + half + k] += 1
        # q / K / V destination: the slot holds whole heads, so the 4 lanes stay in one of them
        seg = 0 if nlo < qd else (1 if nlo < qd + kvd else 2)
        assert seg == (0 if nlo + half + 3 < qd else (1 if nlo + half + 3 < qd + kvd else 2))
    assert np.all(seen == 1)
    # byte offsets of a row's first element are multiples of the row pitches: fp32 qkvd, bf16 qd,
    # the cache row hd; with those, element offsets that are multiples of 4 keep the alignment
    assert (qkvd * 4) % 16 == 0 and (qd * 2) % 8 == 0 and (hd * 2) % 8 == 0 and (half * 4) % 16 == 0


def test_rope_items_match_the_kernel_source():
    import os
    src = open(os.path.join(os.path.dirname(__file__), "..", "token_skip_denoising_b200", "csrc",
                            "fused_layer.cu")).read()
    assert "const int groups = p.qkvd >> 3;" in src and "const int gph = half >> 2;" in src
    assert "const int head = rr / gph;" in src and "pis[e] = (rr - head * gph) * 4;" in src
    assert "nlo[e] = head * p.hd + pis[e];" in src
    assert "if (a.hd % 8 || reinterpret_cast<uintptr_t>(a.rope_cos) % 16" in src
