"""Alternative evaluation orders of the same linear recurrence, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).  These are written
independently of ``mss_oracle.c`` and exist to pin its sequential loop:

* the associative composition of affine steps and the prefix scans built on
  it -- sequential, Blelloch (up-sweep / down-sweep), Hillis-Steele and
  chunked -- which the "Paper: Mamba" course page (section "Code") says are
  tested equal, and whose exactness rests on associativity ("NN Lab: Mamba",
  section "The Associative Property of Linear Recurrence");
* the convolution view of a time-invariant SSM, kernel
  K = (C Bbar, C Abar Bbar, C Abar^2 Bbar, ...) ("Exercises -- State-space
  models (Mamba, S4)", convolutional view and the kernel exercise);
* the lower-triangular (semiseparable) matrix form y = M x with
  M[j, i] = C_j . (Abar_j ... Abar_{i+1}) Bbar_i for i <= j ("Mamba" paper
  review, section "Mamba 2", sequential semiseparable matrix).

Elements of a scan are affine maps h -> a*h + b on one state (``a`` and ``b``
may be numpy arrays, one entry per state).  ``compose(p, q)`` is "apply p,
then q":  (a, b) o (a', b') = (a*a', a'*b + b').  The pages lost this formula
in extraction; this is the plainest reading that makes the scan of the pairs
(Abar_t, Bbar_t x_t) produce the states h_t, and it is checked here by
associativity and by equality with the sequential recurrence.
"""
from __future__ import annotations

import numpy as np

IDENTITY = (1.0, 0.0)


def compose(p, q):
    """Affine map "p then q": h -> a_q*(a_p*h + b_p) + b_q."""
    a_p, b_p = p
    a_q, b_q = q
    return (a_p * a_q, a_q * b_p + b_q)


def scan_sequential(pairs):
    """Inclusive prefix compositions, left to right, one element at a time."""
    out = []
    acc = None
    for p in pairs:
        acc = p if acc is None else compose(acc, p)
        out.append(acc)
    return out


def scan_hillis_steele(pairs):
    """Inclusive scan by Hillis-Steele doubling: log2(L) rounds, at round k
    element i combines with element i - 2^k (work O(L log L))."""
    cur = list(pairs)
    n = len(cur)
    step = 1
    while step < n:
        nxt = list(cur)
        for i in range(step, n):
            nxt[i] = compose(cur[i - step], cur[i])
        cur = nxt
        step *= 2
    return cur


def scan_blelloch(pairs):
    """Inclusive scan by Blelloch's work-efficient method.

    The input is padded to a power of two with the identity.  The up-sweep
    builds a reduction tree in place; the root is replaced by the identity and
    the down-sweep pushes exclusive prefixes back to the leaves.  The inclusive
    result is exclusive prefix o element.  Work O(L), depth O(log L).
    """
    n = len(pairs)
    if n == 0:
        return []
    size = 1
    while size < n:
        size *= 2
    tree = list(pairs) + [IDENTITY] * (size - n)
    # up-sweep: tree[i + 2d - 1] <- tree[i + d - 1] o tree[i + 2d - 1]
    d = 1
    while d < size:
        for i in range(0, size, 2 * d):
            tree[i + 2 * d - 1] = compose(tree[i + d - 1], tree[i + 2 * d - 1])
        d *= 2
    # down-sweep from the root, which starts as the identity
    tree[size - 1] = IDENTITY
    d = size // 2
    while d >= 1:
        for i in range(0, size, 2 * d):
            left = tree[i + d - 1]
            tree[i + d - 1] = tree[i + 2 * d - 1]
            tree[i + 2 * d - 1] = compose(tree[i + 2 * d - 1], left)
        d //= 2
    # tree[i] is now the exclusive prefix of element i
    return [compose(tree[i], pairs[i]) for i in range(n)]


def scan_chunked(pairs, chunk: int):
    """Inclusive scan in chunks: each chunk is scanned on its own from the
    identity, then the running total of the previous chunks (the carry) is
    applied in front of every element of the chunk."""
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    out = []
    carry = None
    for start in range(0, len(pairs), chunk):
        local = scan_sequential(pairs[start:start + chunk])
        if carry is not None:
            local = [compose(carry, p) for p in local]
        out.extend(local)
        carry = local[-1]
    return out


def states_from_scan(prefixes, h0=0.0):
    """h_t = (prefix_t applied to h0) = a_t*h0 + b_t."""
    return [a * h0 + b for (a, b) in prefixes]


def conv_kernel(abar, bbar, c, length: int):
    """Kernel of a time-invariant diagonal SSM:  K_k = sum_n c_n abar_n^k bbar_n."""
    abar = np.asarray(abar, dtype=np.float64)
    bbar = np.asarray(bbar, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    return np.array([np.sum(c * abar ** k * bbar) for k in range(length)])


def causal_conv(kernel, x):
    """y_t = sum_{k=0..t} K_k x_{t-k}  (direct O(L^2) sum)."""
    x = np.asarray(x, dtype=np.float64)
    return np.array([sum(kernel[k] * x[t - k] for k in range(t + 1)) for t in range(len(x))])


def sss_matrix(abar, bbar, c):
    """Materialise M[j, i] = sum_n c[j, n] * (prod_{k=i+1..j} abar[k, n]) * bbar[i, n]
    for i <= j, zero above the diagonal.  abar, bbar, c are [L, N]; then the
    recurrence output is y = M @ x for a scalar input x [L]."""
    abar = np.asarray(abar, dtype=np.float64)
    bbar = np.asarray(bbar, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    L, _ = abar.shape
    M = np.zeros((L, L), dtype=np.float64)
    for j in range(L):
        for i in range(j + 1):
            decay = np.ones(abar.shape[1])
            for k in range(i + 1, j + 1):
                decay = decay * abar[k]
            M[j, i] = np.sum(c[j] * decay * bbar[i])
    return M


# --------------------------------------------------------------------------
# Structured state space duality (scalar A per head): the matrix view and the
# chunked algorithm ("NN Lab -- Mamba", Structured State Space Duality;
# "Mamba" paper review, section "Mamba 2").  One head, fp64, numpy.

def ssd_matrix(a, delta, B, C):
    """The 1-semiseparable matrix of one head: M[j, i] = a_{i+1} ... a_j
    (C_j . B_i) delta_i for i <= j, else 0.  a, delta: [L]; B, C: [L, N]."""
    L = len(a)
    M = np.zeros((L, L))
    for j in range(L):
        prod = 1.0
        for i in range(j, -1, -1):
            M[j, i] = prod * float(C[j] @ B[i]) * delta[i]
            prod *= a[i]
    return M


def ssd_chunked(a, delta, B, C, X, chunk, S0=None):
    """The chunked form: within each chunk the quadratic (attention-like)
    product of the masked M block with X; across chunks the state
    S = (decay of the chunk) S + (the chunk's contribution), carried forward.
    a, delta: [L]; B, C: [L, N]; X: [L, P]; S0: [N, P].  Returns (Y [L, P], S)."""
    L, P = X.shape
    N = B.shape[1]
    S = np.zeros((N, P)) if S0 is None else np.array(S0, dtype=np.float64)
    Y = np.zeros((L, P))
    for c0 in range(0, L, chunk):
        c1 = min(c0 + chunk, L)
        ac, dc, Bc, Cc, Xc = a[c0:c1], delta[c0:c1], B[c0:c1], C[c0:c1], X[c0:c1]
        q = c1 - c0
        # cumulative decay from the chunk start: cum[t] = a_{c0} ... a_{c0+t}
        cum = np.cumprod(ac)
        # intra-chunk: masked quadratic form
        Mc = ssd_matrix(ac, dc, Bc, Cc)
        Y[c0:c1] = Mc @ Xc
        # inter-chunk: the incoming state seen through the decay so far
        Y[c0:c1] += (Cc * cum[:, None]) @ S
        # the chunk's contribution to the state at its end
        tail = np.array([np.prod(ac[t + 1:]) for t in range(q)])
        S = cum[-1] * S + (Bc * (dc * tail)[:, None]).T @ Xc
    return Y, S
