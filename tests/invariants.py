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


def _runs(x):
    """Run symbols, start times and the run index of every position."""
    x = np.asarray(x, np.int64)
    T = len(x)
    start = np.ones(T, bool)
    start[1:] = x[1:] != x[:-1]
    idx = np.cumsum(start) - 1
    st = np.flatnonzero(start)
    return x[st], st, idx


def check_rle_stream(q, k, v, g, end, ln, sym, full=True, sample=None, rng=None):
    """Raise AssertionError on the first violated property of one stream of
    run-level retrieval (adjacent folding): both streams fold into runs of
    equal symbols, the answer is taken at each query run's start time u and
    held over the run, key run l is admissible iff the next key run starts
    at or before u - g + 1, and tau = end + 1 is that next run's start.

    Always (every t): constant over each query run; L = 0 <=> end = -1 <=>
    sym = -1; tau is a key-run start with tau <= u - g + 1; the L query runs
    ending at t's run equal the L key runs ending at the run of tau - 1;
    sym = v[tau].  With ``full`` or at ``sample`` query runs: maximality (no
    admissible key run with a longer run-level match) and recency (no later
    admissible key run with as long a match).
    """
    q = np.asarray(q, np.int64)
    k = np.asarray(k, np.int64)
    v = np.asarray(v, np.int64)
    T = len(q)
    d, u, qrun = _runs(q)
    c, s, krun = _runs(k)
    for t in range(T):
        m = int(qrun[t])
        t0 = int(u[m])
        L, i, y = int(ln[t]), int(end[t]), int(sym[t])
        assert (L, i, y) == (int(ln[t0]), int(end[t0]), int(sym[t0])), f"t={t}: differs from its run start {t0}"
        if L == 0:
            assert i == -1 and y == -1, f"t={t}: L=0 but end={i}, sym={y}"
            continue
        tau = i + 1
        assert 1 <= tau <= t0 - g + 1, f"t={t}: tau={tau} not admissible for the run starting at {t0}"
        assert k[tau] != k[tau - 1], f"t={t}: tau={tau} is not a key-run start"
        assert y == v[tau], f"t={t}: sym={y} != v[tau]={v[tau]}"
        lk = int(krun[tau - 1])
        assert m - L + 1 >= 0 and lk - L + 1 >= 0, f"t={t}: match of {L} runs starts before a stream start"
        assert np.array_equal(d[m - L + 1:m + 1], c[lk - L + 1:lk + 1]), f"t={t}: run symbols differ"
    if full:
        ms = range(len(d))
    elif sample:
        rng = rng or np.random.default_rng(0)
        ms = rng.choice(len(d), size=min(sample, len(d)), replace=False)
    else:
        ms = []
    for m in ms:
        m = int(m)
        t0 = int(u[m])
        L, i = int(ln[t0]), int(end[t0])
        adm = [l for l in range(len(c) - 1) if s[l + 1] <= t0 - g + 1]
        lstar = int(krun[i]) if L > 0 else -1
        for l in adm:
            n = 0
            while n <= m and n <= l and d[m - n] == c[l - n]:
                n += 1
            assert n <= L, f"run {m} (t={t0}): key run {l} matches {n} > {L} runs"
            if L > 0:
                assert not (n == L and l > lstar), f"run {m} (t={t0}): later key run {l} than {lstar}"
