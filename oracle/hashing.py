"""Bigram hash of the decoder-rtx n-gram tables (fp64 oracle; test infrastructure).

Chris McCormick's decoder-rtx posts: "Two huge bi-gram hash tables: 2M rows,
added to x0; 1M rows, added to values".  The row of position t is a hash of
the token pair (x_{t-1}, x_t): key = (a*p1 XOR b*p2) over uint64, row =
key mod rows.  The pages do not give the constants or what precedes the first
token; the readings taken here are p1 = 2654435761, p2 = 2246822519, uint64
wrap-around, and a = vocab (one past the last id) at t = 0.  Both tables use
the same key.
"""

import numpy as np

_MASK64 = (1 << 64) - 1


def bigram_keys(tokens, vocab, p1, p2):
    """uint64 keys [B, T] for int tokens [B, T] (pure Python integers)."""
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    keys = np.zeros((B, T), dtype=np.uint64)
    for b in range(B):
        for t in range(T):
            a = int(tokens[b, t - 1]) if t > 0 else int(vocab)
            c = int(tokens[b, t])
            key = ((a * p1) & _MASK64) ^ ((c * p2) & _MASK64)
            keys[b, t] = np.uint64(key)
    return keys


def bigram_rows(tokens, vocab, p1, p2, n_rows):
    """Table row of every position: key mod n_rows, as int64 [B, T]."""
    keys = bigram_keys(tokens, vocab, p1, p2)
    return np.array([[int(k) % int(n_rows) for k in row] for row in keys],
                    dtype=np.int64).reshape(keys.shape)
