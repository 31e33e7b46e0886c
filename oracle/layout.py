"""Integer token-layout maps of the oracle (test infrastructure only).

Written from "上下文并行与 Ring Attention" (hs-black.github.io):
  * section Ring Attention: at ring step r (from 0) rank i holds the K/V that
    rank (i - r) mod N started with;
  * section 因果掩码带来的负载不均: the contiguous split gives rank i the i-th
    run of c = S/N consecutive tokens;
  * section Zig-zag: the sequence is cut into 2N chunks C_0..C_{2N-1} of c/2
    tokens and rank i takes C_i and C_{2N-1-i} (kept in that order: C_i first);
  * section Striped: token p goes to rank p mod N (local index p // N);
  * section 重排 token 的代价: the mask is judged on original positions, so the
    layouts only permute tokens.

Everything here is plain Python integers; it shares nothing with the product
library's own layout code.
"""

CONTIGUOUS, ZIGZAG, STRIPED = "contiguous", "zigzag", "striped"
LAYOUTS = (CONTIGUOUS, ZIGZAG, STRIPED)


def tokens_per_rank(layout, n_ranks, seq_len):
    if n_ranks <= 0 or seq_len % n_ranks:
        raise ValueError("S must be a multiple of N")
    if layout == ZIGZAG and seq_len % (2 * n_ranks):
        raise ValueError("zig-zag needs S to be a multiple of 2N")
    if layout not in LAYOUTS:
        raise ValueError(layout)
    return seq_len // n_ranks


def position(layout, n_ranks, seq_len, rank, t):
    """Original position of local token t on rank `rank`."""
    c = tokens_per_rank(layout, n_ranks, seq_len)
    if not (0 <= rank < n_ranks and 0 <= t < c):
        raise IndexError((rank, t))
    if layout == CONTIGUOUS:
        return rank * c + t
    if layout == ZIGZAG:
        half = c // 2
        if t < half:
            return rank * half + t
        return (2 * n_ranks - 1 - rank) * half + (t - half)
    return t * n_ranks + rank  # striped


def rank_positions(layout, n_ranks, seq_len, rank):
    c = tokens_per_rank(layout, n_ranks, seq_len)
    return [position(layout, n_ranks, seq_len, rank, t) for t in range(c)]


def rank_order(layout, n_ranks, seq_len):
    """order[i*c + t] = original position of local token t on rank i."""
    out = []
    for i in range(n_ranks):
        out.extend(rank_positions(layout, n_ranks, seq_len, i))
    return out


def ring_source(rank, step, n_ranks):
    """Rank whose K/V block rank `rank` holds at ring step `step`."""
    return (rank - step) % n_ranks


def permute(x, layout, n_ranks, axis):
    """Gather the sequence axis of numpy array x into rank-major order."""
    import numpy as np
    order = np.asarray(rank_order(layout, n_ranks, x.shape[axis]), dtype=np.int64)
    return np.take(x, order, axis=axis)


def unpermute(x_ranked, layout, n_ranks, axis):
    """Inverse of permute: scatter rank-major rows back to original order."""
    import numpy as np
    order = np.asarray(rank_order(layout, n_ranks, x_ranked.shape[axis]), dtype=np.int64)
    out = np.empty_like(x_ranked)
    idx = [slice(None)] * x_ranked.ndim
    idx[axis] = order
    out[tuple(idx)] = x_ranked
    return out


def visible_pairs(layout, n_ranks, seq_len, rank, src, causal=True):
    """Brute-force count of (query, key) pairs of rank `rank` against rank `src`'s
    tokens that the causal mask leaves visible (pos_k <= pos_q)."""
    pq = rank_positions(layout, n_ranks, seq_len, rank)
    pk = rank_positions(layout, n_ranks, seq_len, src)
    if not causal:
        return len(pq) * len(pk)
    return sum(1 for a in pq for b in pk if b <= a)


def chunk_pair_kind(n_ranks, q_chunk, k_chunk, chunk_len=4):
    """Kind of one (query chunk, key chunk) pair under the causal mask, found by
    enumerating positions: 'full', 'diag' (partly visible) or 'skip'."""
    qs = range(q_chunk * chunk_len, (q_chunk + 1) * chunk_len)
    ks = range(k_chunk * chunk_len, (k_chunk + 1) * chunk_len)
    vis = sum(1 for a in qs for b in ks if b <= a)
    if vis == 0:
        return "skip"
    if vis == chunk_len * chunk_len:
        return "full"
    return "diag"
