"""Frozen trigram statistics table projected into the values (fp64 oracle;
test infrastructure only, see oracle/__init__.py).

Chris McCormick's decoder-rtx posts (baseline 4) add "a 2M row tri-gram stats
table (tallied from dataset, frozen), projected and added to values" and say
no more.  The readings taken here, each the plainest one the rest of the
pages support:

  * row of position t: a hash of the token triple (x_{t-2}, x_{t-1}, x_t) in
    the form of the bigram tables' hash, key = (a2*p1 XOR a1*p2 XOR c*p3) over
    uint64 with p3 = 3266489917, the vocabulary size standing for the tokens
    before the start of a sequence; row = key mod rows;
  * "stats tallied from dataset": for every position t of a token stream that
    has a next token, the row of t counts the next token in bucket
    (x_{t+1} mod width); a row's statistics are its counts over its total
    (the empirical next-token distribution folded into `width` buckets), a
    row never seen stays zero;
  * "frozen": no gradient reaches the table;
  * "projected and added to values": a learned matrix vproj [H*hd, width]
    maps a position's statistics into the value space, v_t += vproj s_row(t),
    in every layer (the same term, like the value table), so its gradient is
    the value gradient summed over layers times the statistics.
"""

import numpy as np

_MASK64 = (1 << 64) - 1
P3 = 3266489917


def trigram_keys(tokens, vocab, p1, p2, p3=P3):
    """uint64 keys [B, T] of int tokens [B, T] (pure Python integers)."""
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    keys = np.zeros((B, T), dtype=np.uint64)
    for b in range(B):
        for t in range(T):
            a2 = int(tokens[b, t - 2]) if t > 1 else int(vocab)
            a1 = int(tokens[b, t - 1]) if t > 0 else int(vocab)
            c = int(tokens[b, t])
            key = ((a2 * p1) & _MASK64) ^ ((a1 * p2) & _MASK64) ^ ((c * p3) & _MASK64)
            keys[b, t] = np.uint64(key)
    return keys


def trigram_rows(tokens, vocab, p1, p2, n_rows, p3=P3):
    """Table row of every position: key mod n_rows, as int64 [B, T]."""
    keys = trigram_keys(tokens, vocab, p1, p2, p3)
    return np.array([[int(k) % int(n_rows) for k in row] for row in keys],
                    dtype=np.int64).reshape(keys.shape)


def tally_counts(streams, vocab, p1, p2, n_rows, width, p3=P3):
    """Counts of the tally: (rows [U] ascending, counts [U, width] int64) over
    the rows that occur.  streams [S, L]: position t < L - 1 of each stream
    counts its next token x_{t+1} in bucket x_{t+1} mod width of its row."""
    streams = np.asarray(streams)
    rows = trigram_rows(streams, vocab, p1, p2, n_rows, p3)[:, :-1].reshape(-1)
    buckets = (streams[:, 1:] % width).reshape(-1)
    uniq = np.unique(rows)
    counts = np.zeros((len(uniq), width), dtype=np.int64)
    np.add.at(counts, (np.searchsorted(uniq, rows), buckets), 1)
    return uniq, counts


def tally_stats(streams, vocab, p1, p2, n_rows, width, p3=P3):
    """The statistics of the rows that occur: (rows [U], stats [U, width]),
    each row's counts over its total."""
    uniq, counts = tally_counts(streams, vocab, p1, p2, n_rows, width, p3)
    return uniq, counts / counts.sum(axis=1, keepdims=True)


def dense_stats(streams, vocab, p1, p2, n_rows, width, p3=P3):
    """The whole [n_rows, width] table (small tables only)."""
    uniq, stats = tally_stats(streams, vocab, p1, p2, n_rows, width, p3)
    table = np.zeros((n_rows, width))
    table[uniq] = stats
    return table
