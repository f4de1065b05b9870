"""Independent checks of retrieval outputs, used to pin the oracle and the
CUDA path.  Written from the definition (longest admissible suffix match,
most recent end, sym = v[i+1]); they share no code with either matcher."""
import numpy as np


def check_stream(q, k, v, g, end, ln, sym, full=True, sample=None, rng=None):
    """Raise AssertionError on the first violated property of one stream.

    Always (every t): L_t <= L_{t-1} + 1; i <= t - g; L = 0 <=> i = -1;
    q[t-L+1..t] == k[i-L+1..i]; sym = v[i+1].
    With ``full`` (O(T^2)) or at ``sample`` positions: maximality (no
    admissible occurrence of length L+1) and recency (no occurrence of
    length L ending in (i, t-g]).
    """
    T = len(q)
    q = np.asarray(q, np.int64)
    k = np.asarray(k, np.int64)
    v = np.asarray(v, np.int64)
    prev = 0
    for t in range(T):
        L, i, s = int(ln[t]), int(end[t]), int(sym[t])
        assert L <= prev + 1, f"t={t}: L={L} > L_prev+1={prev + 1}"
        prev = L
        if L == 0:
            assert i == -1 and s == -1, f"t={t}: L=0 but i={i}, sym={s}"
            continue
        assert 0 <= i <= t - g, f"t={t}: i={i} not admissible (g={g})"
        assert i - L + 1 >= 0, f"t={t}: match runs before the key start"
        assert np.array_equal(q[t - L + 1:t + 1], k[i - L + 1:i + 1]), f"t={t}: substrings differ"
        assert s == v[i + 1], f"t={t}: sym={s} != v[i+1]={v[i + 1]}"
    if full:
        ts = range(T)
    elif sample:
        rng = rng or np.random.default_rng(0)
        ts = rng.choice(T, size=min(sample, T), replace=False)
    else:
        ts = []
    for t in ts:
        t = int(t)
        L, i = int(ln[t]), int(end[t])
        hi = t - g
        if hi < 0:
            assert L == 0
            continue
        # maximality: no admissible end j with k[j-L..j] == q[t-L..t]
        if L + 1 <= t + 1:
            pat = q[t - L:t + 1]
            for j in range(L, hi + 1):
                assert not np.array_equal(k[j - L:j + 1], pat), f"t={t}: longer match ends at {j}"
        if L == 0:
            continue
        pat = q[t - L + 1:t + 1]
        for j in range(i + 1, hi + 1):
            if j - L + 1 >= 0:
                assert not np.array_equal(k[j - L + 1:j + 1], pat), f"t={t}: later end {j} than {i}"
