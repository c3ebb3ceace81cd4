"""Index sets of the two access views over one retained KV cache.

[notes §2.1, eq. S^F / S^L]: S^F_t = {1, ..., t};
S^L_t = {1, ..., min(s, t)} U {max(1, t - w + 1), ..., t}, with s = 4 initial (sink)
positions and a w = 2048 recent window that includes the current position t.
Positions are 1-based as on the page; the sets are Python sets (a union: an overlap of
sinks and window counts once).
"""

SINKS = 4
WINDOW = 2048


def full_set(t: int) -> set:
    """S^F_t = {1..t}."""
    if t < 1:
        raise ValueError("t must be >= 1")
    return set(range(1, t + 1))


def local_set(t: int, s: int = SINKS, w: int = WINDOW) -> set:
    """S^L_t = {1..min(s,t)} U {max(1, t-w+1)..t}."""
    if t < 1:
        raise ValueError("t must be >= 1")
    return set(range(1, min(s, t) + 1)) | set(range(max(1, t - w + 1), t + 1))
