"""Independent recomputation of the decode plan's split partition (host-only
test helper: no GPU, no library code)."""

SEGMENT_COST_PAGES = 4  # places a sequence boundary takes on the partition's cost line


def reference_segments(lens, P, W):
    """Independent recomputation of the split partition: lay the pages out on a
    cost line where each sequence boundary takes SEGMENT_COST_PAGES places, cut
    the line into W equal parts (floor), and start each worker at the first
    real page at or after its cut (brute force over the pages)."""
    pages = [-(-x // P) for x in lens]
    bounds = [0]
    for n in pages:
        bounds.append(bounds[-1] + n)
    G = bounds[-1]
    pos = []  # cost-line position of every real page
    for b, n in enumerate(pages):
        pos.extend(bounds[b] + i + SEGMENT_COST_PAGES * b for i in range(n))
    line = G + SEGMENT_COST_PAGES * (len(pages) - 1)

    def start(w):
        cut = w * line // W
        return next((x for x, v in enumerate(pos) if v >= cut), G)

    segs = []
    for w in range(W):
        a, e = start(w), start(w + 1)
        for b in range(len(lens)):
            lo, hi = max(a, bounds[b]), min(e, bounds[b + 1])
            if lo < hi:
                segs.append((w, b, lo - bounds[b], hi - bounds[b], w + b))
    return segs, pages


def segment_key_ranges(lens, P, W, b):
    """The (first key, end key) ranges of sequence b's segments, in key order."""
    segs, _ = reference_segments(lens, P, W)
    return [(s[2] * P, min(s[3] * P, lens[b])) for s in segs if s[1] == b]
