"""Host model of the split-KV partition the device planner computes.

The library decides, on the GPU and from seq_lens alone, which CTA handles
which 64-token blocks.  This module restates that decision in plain Python so
tests can check the device planner bit for bit, and so users can predict the
workspace a call needs.

Flattened work list: sequences b in order; inside b its units (one KV head,
or one chunk of the query heads sharing it) in order; inside a unit the
visible blocks [first_b, last_b] in order, where the visible key range is
[lo_b, T_b) with lo_b = max(0, T_b - window) for window > 0, else 0, and only
blocks holding a visible key are listed.  CTA i of P takes the block range
[floor(i W / P'), floor((i + 1) W / P')) for i < P' = min(P, W); the other
CTAs have no work.
"""
BLOCK_SIZE = 64


def visible_blocks(T, window, max_blocks):
    """(first logical block, number of visible blocks) of one sequence."""
    if T <= 0 or T > max_blocks * BLOCK_SIZE:
        return 0, 0
    lo = T - window if (window > 0 and T > window) else 0
    first = lo // BLOCK_SIZE
    return first, (T - 1) // BLOCK_SIZE - first + 1


def working_ctas(W, P):
    """CTAs that take work: min(P, W), so no working CTA has an empty range."""
    return min(P, W)


def cta_bound(i, W, P):
    return (i * W) // P


def plan(seq_lens, units_per_seq, window, max_blocks, num_ctas):
    """Same layout as attn_decode_plan: [W, (lo, hi, seq, unit) * P, prefix]."""
    work = [visible_blocks(int(T), window, max_blocks)[1] * units_per_seq
            for T in seq_lens]
    prefix = [0]
    for w in work:
        prefix.append(prefix[-1] + w)
    W = prefix[-1]
    P = working_ctas(W, num_ctas)
    out = [W]
    for i in range(num_ctas):
        lo = cta_bound(i, W, P) if i < P else W
        hi = cta_bound(i + 1, W, P) if i < P else W
        if lo >= hi:
            out += [lo, hi, -1, -1]
            continue
        b = max(j for j in range(len(work)) if work[j] > 0 and prefix[j] <= lo)
        nb = work[b] // units_per_seq
        out += [lo, hi, b, (lo - prefix[b]) // nb]
    return out + prefix


def cta_of(x, W, P):
    """The CTA whose range holds flattened block x."""
    i = (x * P) // W
    while i + 1 < P and cta_bound(i + 1, W, P) <= x:
        i += 1
    while i > 0 and cta_bound(i, W, P) > x:
        i -= 1
    return i


def splits_of_unit(seq_lens, units_per_seq, window, max_blocks, num_ctas, b,
                   unit):
    """CTAs (in order) that hold a part of (sequence b, unit)."""
    p = plan(seq_lens, units_per_seq, window, max_blocks, num_ctas)
    W = p[0]
    prefix = p[1 + 4 * num_ctas:]
    nb = visible_blocks(int(seq_lens[b]), window, max_blocks)[1]
    if nb == 0:
        return []
    s = prefix[b] + unit * nb
    P = working_ctas(W, num_ctas)
    return list(range(cta_of(s, W, P), cta_of(s + nb - 1, W, P) + 1))
