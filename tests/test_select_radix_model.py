"""The select kernel's radix passes on raw float bits, modelled on the host: the histogram of each
8-bit digit is counted on the raw bits of (score + 0.0) and read back in the order of the
order-preserving key (first digit: non-negative raw bytes 0..127 are key bins 128..255, negative
raw bytes 128..255 are key bins 127..0; later digits of a negative prefix run in reverse), and a
later pass counts a score in bin min((raw ^ raw_prefix) >> shift, 256), bin 256 being the spare
slot. This checks that arithmetic (not the CUDA code) against a plain sort by (score desc, index
asc) on inputs with negative thresholds, signed zeros, subnormals, exact ties and wide ranges,
where the radix passes go down to the last digit."""
import numpy as np
import pytest


def key_of(raw: np.ndarray) -> np.ndarray:
    """Order-preserving key of raw fp32 bits (non-negative: set the sign bit; negative: invert)."""
    raw = raw.astype(np.uint32)
    return np.where(raw >> 31, ~raw, raw | np.uint32(0x80000000)).astype(np.uint32)


def raw_prefix(prefix: int, mask: int) -> int:
    return (prefix ^ 0x80000000) if prefix & 0x80000000 else (~prefix & mask) & 0xFFFFFFFF


def raw_bin(kb: int, first: bool, neg: bool) -> int:
    if first:
        return kb - 128 if kb >= 128 else 255 - kb
    return 255 - kb if neg else kb


def threshold_by_raw_passes(scores: np.ndarray, m: int):
    """(prefix, mask, rem, nb) after the histogram passes, as the kernel resolves them."""
    raw = (scores.astype(np.float32) + np.float32(0.0)).view(np.uint32)
    prefix = mask = 0
    rem, nb = m, len(scores)
    done = rem == nb
    for p in range(4):
        if done:
            break
        shift = 24 - 8 * p
        if p == 0:
            idx = (raw >> np.uint32(24)).astype(np.int64)
        else:
            rp = np.uint32(raw_prefix(prefix, mask))
            idx = np.minimum((raw ^ rp) >> np.uint32(shift), np.uint32(256)).astype(np.int64)
        hist = np.bincount(idx, minlength=257)
        above = 0
        neg = (prefix & 0x80000000) == 0
        for kb in range(255, -1, -1):
            h = int(hist[raw_bin(kb, p == 0, neg)])
            if above + h >= rem:
                prefix |= kb << shift
                mask |= 0xFF << shift
                rem -= above
                nb = h
                break
            above += h
        else:
            raise AssertionError(f"pass {p}: no bin holds the m-th key")
        done = rem == nb or mask == 0xFFFFFFFF
    return prefix, mask, rem, nb


def select_by_raw_passes(scores: np.ndarray, m: int) -> np.ndarray:
    """Indices of the m best: keys above the resolved bucket, then the bucket's keys by (key desc,
    index asc) up to rem (the kernel takes the bucket whole, its exact ties in index order, or
    collects it and ranks it exactly)."""
    keys = key_of((scores.astype(np.float32) + np.float32(0.0)).view(np.uint32))
    prefix, mask, rem, nb = threshold_by_raw_passes(scores, m)
    hi = prefix | (~mask & 0xFFFFFFFF)
    above = np.nonzero(keys > np.uint32(hi))[0]
    bucket = np.nonzero((keys >= np.uint32(prefix)) & (keys <= np.uint32(hi)))[0]
    assert len(bucket) == nb and len(above) + rem == m
    order = np.lexsort((bucket, -keys[bucket].astype(np.int64)))
    return np.sort(np.concatenate([above, bucket[order[:rem]]]))


def select_by_sort(scores: np.ndarray, m: int) -> np.ndarray:
    s = scores.astype(np.float32) + np.float32(0.0)
    order = np.lexsort((np.arange(len(s)), -s.astype(np.float64)))
    return np.sort(order[:m])


def cases():
    rng = np.random.default_rng(7)
    yield "normal", rng.standard_normal(3000).astype(np.float32), 511
    yield "mostly_negative", (rng.standard_normal(2000) - 4.0).astype(np.float32), 1500
    z = np.zeros(1200, dtype=np.float32)
    z[::2] = -0.0
    z[::7] = rng.standard_normal(len(z[::7])).astype(np.float32)
    yield "signed_zeros", z, 600
    yield "subnormals", (rng.standard_normal(1500) * 1e-40).astype(np.float32), 700
    ties = rng.integers(-3, 4, 4000).astype(np.float32)
    yield "exact_ties", ties, 2047
    wide = (rng.standard_normal(3000) * np.exp(rng.uniform(-60, 60, 3000))).astype(np.float32)
    yield "wide_range", wide, 1000
    near = (np.float32(150.0) + rng.integers(-3, 4, 5000).astype(np.float32) * np.float32(2.0 ** -16)).astype(np.float32)
    yield "last_digit", near, 2500
    yield "negative_last_digit", -near, 2500


@pytest.mark.parametrize("name,scores,m", list(cases()), ids=[c[0] for c in cases()])
def test_raw_bit_radix_select_matches_sort(name, scores, m):
    np.testing.assert_array_equal(select_by_raw_passes(scores, m), select_by_sort(scores, m))


def test_first_digit_maps_key_order():
    """Key bins in descending order visit the raw bytes from the largest score down."""
    vals = np.array([np.inf, 3.0, 1.0, 0.0, -0.0, -1.0, -3.0, -np.inf], dtype=np.float32)
    raw_top = ((vals + np.float32(0.0)).view(np.uint32) >> np.uint32(24)).tolist()
    order = [raw_bin(kb, True, False) for kb in range(255, -1, -1)]
    pos = [order.index(b) for b in raw_top]
    assert pos == sorted(pos)


def test_emit_raw_comparisons_match_key_comparisons():
    """The emit pass's fast path for thresholds above the key of +0.0 compares raw bits (no +0.0
    add): (int32) raw >= (int32) (thr ^ 2^31) must equal key >= thr, and (raw - (blo ^ 2^31))
    mod 2^32 <= bw must equal blo <= key <= blo + bw (blo at or above the key of +0.0), for every
    score, -0.0 and negative ones included."""
    rng = np.random.default_rng(11)
    scores = np.concatenate([rng.standard_normal(4000).astype(np.float32) * 300,
                             np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45], dtype=np.float32)])
    raw = scores.view(np.uint32)
    keys = key_of((scores + np.float32(0.0)).view(np.uint32)).astype(np.int64)
    raw_s = raw.view(np.int32).astype(np.int64)
    thrs = np.concatenate([keys[keys > 0x80000000][:200], [0x80000001, 0xFF800000, 0xFFFFFFFF]])
    for thr in thrs.astype(np.int64):
        fast = raw_s >= np.int64(np.uint32(thr ^ 0x80000000).view(np.int32))
        np.testing.assert_array_equal(fast, keys >= thr)
    for blo in thrs[:100].astype(np.int64):
        for bw in (0, 1, 0xFF, 0xFFFF):
            if blo + bw > 0xFFFFFFFF:
                continue
            fast = ((raw.astype(np.int64) - (blo ^ 0x80000000)) % (1 << 32)) <= bw
            np.testing.assert_array_equal(fast, (keys >= blo) & (keys <= blo + bw))
