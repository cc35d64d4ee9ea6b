"""CPU oracle for one MoE layer: route -> balance -> dispatch -> expert FFN -> combine.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or executes this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may.  It shares no code with the CUDA library (no kernels, headers,
helpers, tables or constants); both sides get their inputs from the seeded generators in
``load_balanced_dispatch_warp_b200/inputs.py``.

Every function is the plain definition of its step, written slowly and in fp64 for
floating point, citing the page passage it follows.  Sources (page title, section):

  [MoonEP]   "Moonshot AI drops MoonEP, claims 2.5x scaling boost for trillion-parameter
             models" -- news article; para. 2 (maxvio), para. 3 (equal-load invariant,
             redundant copies planned from router output, prefetch, zero-copy placement,
             static shapes, one process-global pool), para. 4 (slot policy).
  [Primer]   "DeepEP-on-EFA Guidance, section 1: What is MoE" -- the four-phase EP
             pipeline: (a) router/top-k, (b) dispatch, (c) expert FFN as grouped GEMM,
             (d) combine = transpose of dispatch, gate-weighted sum.
  [Hotspots] "MoE Load Balancing: Find Expert Hotspots" -- sections "Separate expert
             demand from rank placement", "Make expert capacity, overflow, and padding
             explicit", "Count remote routes before celebrating balance", "Work the
             16-token hotspot fixture", "Reject incomparable MoE load-balancing traces".

Pins (tests/test_oracle_pins.py checks each against something other than this file):
  topk_route        brute-force rank counting on tiny inputs; k=1 / k=E special cases;
                    softmax closed forms (k=2 sigmoid, equal logits -> 1/k)
  topk_route_biased zero bias reduces to topk_route; a large bias forces a chosen set;
                    the gates ignore the bias, equal or unequal on the chosen pair
                    (closed form for k=2)
  expert_histogram  the pages' worked fixture (demand, both rank mappings, 4/9, 8/15, 0.8)
  capacity_ledger   the pages' worked fixture (cap 5, processed/overflow/padding)
  remote_routes     the pages' worked fixture (22 vs 25 of 32)
  plan_balanced     invariants (exact per-rank load, every assignment once, replica
                    accounting) over exhaustive tiny inputs, plus a plan derived by hand
                    for the fixture.  WHICH valid plan is chosen is not fixed by the pages
                    (they give no algorithm): that choice is this oracle's reading.
  permute/dispatch  bijection and x-row identity checks on random inputs
  prefetch          bitwise slot = home-expert identity
  expert_ffn        closed forms: identity / single-entry weights give silu(a)*a with
                    silu(1) = e/(1+e); transposed operands land in distinct outputs
  combine           identity experts return x (gates sum to one); per-expert scaling
                    returns (sum_j gate_j c_e) x; dropped assignments (perm = -1) add
                    nothing
  dispatch_capacity the pages' worked fixture at cap 5 (processed [5,5,5,4,3,2,2,1],
  layer_capacity    overflow [4,1,0,...], padding 13, the dropped assignments derived by
                    hand); a capacity above every demand reduces to the dropless layer;
                    identity experts return (sum of kept gates) x
  ep_local_counts, ep_rank_base, ep_permute, ep_layer
                    W processes computing the undistributed layer() of the rank-major
                    concatenated batch (same perm, the same rows on every rank, the same
                    outputs); q_base counted directly on the concatenated trace; one
                    rank's error reaches the job's error word
  ep_layer_backward the W-process backward equals layer_backward() of the concatenated
                    batch (dx, dlogits, dy and dX rows per rank, every weight gradient)
  layer_backward    central finite differences of layer() itself (fp64, tiny shapes,
                    away from top-k ties); torch.autograd (fp64, CPU) through a token-major
                    formulation with no plan, dispatch or replicas; the weight gradients do
                    not depend on S (replicas reduced back home)
  dispatch_backward, combine_backward
                    the adjoint (dot-product) identity <A v, w> = <v, A^T w> against
                    dispatch() and combine() on random inputs, for the rows and the gates
  topk_backward     central differences of topk_route's gates along fp32-exact directions
  expert_ffn_backward  central differences of expert_ffn() for X, w1, w3, w2
  (tests/test_oracle_mutants.py plants one plausible mistake at a time in topk_route,
  topk_route_biased, validate_trace, expert_histogram, capacity_ledger, remote_routes,
  plan_balanced, permute, dispatch, prefetch, expert_ffn, combine, ep_rank_base,
  ep_permute, ep_layer_backward and the four backward pieces, and checks that the pin for
  it fails)

Error bits (OR-ed): 1 non-finite logit, 2 expert id out of range, 4 repeated expert
within one token, 8 plan needs more than S replicas on some rank.
"""
from __future__ import annotations

import numpy as np

ERR_NONFINITE = 1
ERR_ID_RANGE = 2
ERR_DUPLICATE = 4
ERR_SLOTS = 8


# --------------------------------------------------------------------------- (a) router
def topk_route(logits: np.ndarray, k: int):
    """Top-k expert choice and gate weights per token  ([Primer] phase (a) router).

    For each token the (logit, expert) pairs are ordered by logit descending, ties by
    the lower expert id first, and the first k are taken.  The gate of the j-th choice
    is the softmax over the k selected logits:
        gate_j = exp(l_j - l_max) / sum_{i in top-k} exp(l_i - l_max)
    computed in fp64 from the fp32 logits, so the weights are finite, non-negative and
    sum to one ([Hotspots] "starts with one route trace": finite non-negative weights).
    A non-finite logit anywhere sets error bit 1; that token's outputs are unspecified.

    Returns idx [T,k] int32, gate [T,k] float64, err int.
    """
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    err = 0
    if not np.all(np.isfinite(logits)):
        err |= ERR_NONFINITE
    idx = np.zeros((T, k), dtype=np.int32)
    gate = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        row = logits[t].astype(np.float64)
        if not np.all(np.isfinite(row)):
            continue
        # stable sort on -logit keeps equal logits in ascending expert order
        order = np.argsort(-row, kind="stable")[:k]
        idx[t] = order
        sel = row[order]
        ex = np.exp(sel - sel[0])
        gate[t] = ex / ex.sum()
    return idx, gate, err


def topk_route_biased(logits: np.ndarray, bias: np.ndarray, k: int):
    """Bias-only balancing ("Your MoE router sends 90% of tokens to 10% of the experts":
    a per-expert bias outside the gradient path, as DeepSeek-V3 used, balances the load
    without distorting the gate).  The experts are chosen by the top-k of the biased
    scores s_e = logit_e + bias_e -- the sum taken in fp32, the precision the kernel
    decides in -- ordered by s descending, ties by the lower expert id; the gate of each
    chosen expert is the softmax over the chosen experts' UNBIASED logits, in the chosen
    order, in fp64.  A non-finite logit or bias sets error bit 1.

    Returns idx [T,k] int32, gate [T,k] float64, err int.
    """
    logits = np.asarray(logits, dtype=np.float32)
    bias = np.asarray(bias, dtype=np.float32)
    T, E = logits.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    err = 0
    if not (np.all(np.isfinite(logits)) and np.all(np.isfinite(bias))):
        err |= ERR_NONFINITE
    idx = np.zeros((T, k), dtype=np.int32)
    gate = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        if not (np.all(np.isfinite(logits[t])) and np.all(np.isfinite(bias))):
            continue
        scores = (logits[t] + bias).astype(np.float32)  # fp32 sum, elementwise
        order = np.argsort(-scores.astype(np.float64), kind="stable")[:k]
        idx[t] = order
        sel = logits[t][order].astype(np.float64)
        m = sel.max()
        ex = np.exp(sel - m)
        gate[t] = ex / ex.sum()
    return idx, gate, err


# ------------------------------------------------------------------ demand and imbalance
def home_rank_map(E: int, R: int) -> np.ndarray:
    """Contiguous expert->rank ownership e -> floor(e / (E/R)): rank r owns experts
    [rB, (r+1)B), as in the fixture's initial placement {0,1},{2,3},{4,5},{6,7}
    ([Hotspots] "Separate expert demand from rank placement")."""
    B = E // R
    return (np.arange(E) // B).astype(np.int64)


def validate_trace(idx: np.ndarray, E: int) -> int:
    """Trace validation before anything is sized from it ([Hotspots] "Work the 16-token
    hotspot fixture": ids must be known experts, no token may repeat an expert).
    Returns error bits 2 (id outside [0,E)) and 4 (repeat within a token)."""
    err = 0
    for row in np.asarray(idx):
        ids = [int(v) for v in row]
        if any(v < 0 or v >= E for v in ids):
            err |= ERR_ID_RANGE
        if len(set(ids)) != len(ids):
            err |= ERR_DUPLICATE
    return err


def expert_histogram(idx: np.ndarray, E: int, R: int, expert_to_rank=None):
    """Expert demand, rank demand and the imbalance scalars.

    [Hotspots] "Separate expert demand from rank placement": first count assignments by
    expert, then sum those counts over an expert->rank mapping.  Balancedness is
    average / maximum.  [MoonEP] para. 2: maxvio is 0 when perfectly balanced; adopted as
    (max rank load - mean) / mean.  With A = T*k assignments and mean = A/R this is the
    exact rational (R*max - A) / A, rounded once to fp64; balancedness = A / (R*max).
    Expert-level maxvio uses E buckets instead of R.  Only in-range ids are counted;
    bad ids set the validation error bits.  A = 0 gives maxvio 0 and balancedness 1.

    The mapping is validated too ("Work the 16-token hotspot fixture": if an expert is
    missing from a mapping, stop): an entry outside [0, R) -- no owning rank -- sets
    error bit 2, and that expert's demand is added to no rank (never Python's negative
    indexing, which would hand -1 to rank R-1).

    Returns dict(counts[E], loads[R], maxvio, balancedness, expert_maxvio,
    expert_balancedness, err).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    A = T * k
    err = validate_trace(idx, E)
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if 0 <= e < E:
                counts[e] += 1
    if expert_to_rank is None:
        expert_to_rank = home_rank_map(E, R)
    loads = np.zeros(R, dtype=np.int64)
    for e in range(E):
        r = int(expert_to_rank[e])
        if 0 <= r < R:
            loads[r] += counts[e]
        else:
            err |= ERR_ID_RANGE
    mx = int(loads.max()) if R > 0 else 0
    emx = int(counts.max()) if E > 0 else 0
    if A == 0 or mx == 0:
        maxvio, bal = 0.0, 1.0
    else:
        maxvio = float(R * mx - A) / float(A)
        bal = float(A) / float(R * mx)
    if A == 0 or emx == 0:
        emaxvio, ebal = 0.0, 1.0
    else:
        emaxvio = float(E * emx - A) / float(A)
        ebal = float(A) / float(E * emx)
    return dict(counts=counts, loads=loads, maxvio=maxvio, balancedness=bal,
                expert_maxvio=emaxvio, expert_balancedness=ebal, err=err)


def capacity_ledger(counts, A: int, E: int, cf_num: int = 5, cf_den: int = 4):
    """Fixed-capacity ledger ([Hotspots] "Make expert capacity, overflow, and padding
    explicit"): cap = ceil(A / E * cf) per expert, processed = min(count, cap),
    overflow = max(count - cap, 0), padding = max(cap - count, 0).  The capacity
    factor is an exact rational cf_num/cf_den so the ceiling is exact."""
    num = A * cf_num
    den = E * cf_den
    cap = -(-num // den)
    counts = np.asarray(counts, dtype=np.int64)
    processed = np.minimum(counts, cap)
    overflow = np.maximum(counts - cap, 0)
    padding = np.maximum(cap - counts, 0)
    return dict(cap=int(cap), processed=processed, overflow=overflow, padding=padding)


def remote_routes(idx, origin, expert_to_rank) -> int:
    """Remote-route count ([Hotspots] "Count remote routes before celebrating balance"):
    an assignment is remote when the token's origin rank differs from the rank that
    owns its chosen expert."""
    n = 0
    for t, row in enumerate(np.asarray(idx)):
        for e in row:
            if int(expert_to_rank[int(e)]) != int(origin[t]):
                n += 1
    return n


# ------------------------------------------------------------------ equal-load plan
def plan_balanced(counts, T: int, k: int, E: int, R: int, S: int):
    """Equal-load plan with redundant expert copies ([MoonEP] para. 3-4).

    The article fixes the contract -- every rank receives exactly the same number of
    rows, C = T*k/R, by placing a few redundant expert copies planned from the router
    output, each copy occupying one of S prefetch slots per rank -- but gives no
    algorithm.  The reading used here ("keep small, stream the rest"):

      1. Rank r owns experts [rB, (r+1)B), B = E/R.
      2. Per rank, order its experts by (count ascending, id ascending).  With room = C,
         keep each expert whole while its count fits the room (room -= count); the first
         expert that does not fit and every later one are streamed.  room_r is what is
         left.
      3. The stream is the streamed experts in (home rank, id) order, each expert's
         assignments in token order.  Sum(room_r) equals the stream length.
      4. The ranks' rooms, concatenated in rank order, cut the stream: position p goes to
         the rank u with room_prefix[u] <= p < room_prefix[u+1].
      5. In rank u's piece, each maximal run of one expert whose home is not u is a
         replica; replicas take slots 0, 1, ... of rank u in order.  More than S sets
         error bit 8.
      6. Rank u's rows: [0, kept_u) hold its kept experts in id order (each contiguous),
         [kept_u, C) hold its stream piece in stream order.
      7. Groups are those runs in that order, empty ones left out.  weight_ref = e for an
         expert at its home rank, E + u*S + s for replica slot s of rank u.

    Returns a dict with C, kept_rows[R], room_prefix[R+1], expert_home_off[E] (local
    row offset of a kept expert, -1 if streamed), stream_off[E+1] (exclusive prefix of
    streamed counts in id order), replica_expert[R*S] (-1 empty), groups (list per rank
    of (row_start_global, rows, expert, weight_ref)), err.
    """
    counts = [int(c) for c in counts]
    A = T * k
    assert A % R == 0 and E % R == 0
    C = A // R
    B = E // R
    kept = [False] * E
    kept_rows = [0] * R
    room = [0] * R
    for r in range(R):
        home = list(range(r * B, (r + 1) * B))
        order = sorted(home, key=lambda e: (counts[e], e))
        left = C
        for e in order:
            if counts[e] <= left:
                kept[e] = True
                left -= counts[e]
            else:
                break
        room[r] = left
        kept_rows[r] = C - left
    room_prefix = [0] * (R + 1)
    for r in range(R):
        room_prefix[r + 1] = room_prefix[r] + room[r]
    stream_off = [0] * (E + 1)
    for e in range(E):
        stream_off[e + 1] = stream_off[e] + (0 if kept[e] else counts[e])
    assert stream_off[E] == room_prefix[R]
    expert_home_off = [-1] * E
    for r in range(R):
        off = 0
        for e in range(r * B, (r + 1) * B):
            if kept[e]:
                expert_home_off[e] = off
                off += counts[e]
    replica_expert = [-1] * (R * S)
    groups = [[] for _ in range(R)]
    err = 0
    for u in range(R):
        for e in range(u * B, (u + 1) * B):
            if kept[e] and counts[e] > 0:
                groups[u].append((u * C + expert_home_off[e], counts[e], e, e))
        lo, hi = room_prefix[u], room_prefix[u + 1]
        n_rep = 0
        for e in range(E):
            if kept[e] or counts[e] == 0:
                continue
            a, b = max(lo, stream_off[e]), min(hi, stream_off[e] + counts[e])
            if a >= b:
                continue
            row = u * C + kept_rows[u] + (a - lo)
            if e // B == u:
                groups[u].append((row, b - a, e, e))
            else:
                if n_rep < S:
                    replica_expert[u * S + n_rep] = e
                    groups[u].append((row, b - a, e, E + u * S + n_rep))
                n_rep += 1
        if n_rep > S:
            err |= ERR_SLOTS
    return dict(C=C, kept=kept, kept_rows=kept_rows, room_prefix=room_prefix,
                expert_home_off=expert_home_off, stream_off=stream_off,
                replica_expert=replica_expert, groups=groups, err=err)


# ------------------------------------------------------------------ placement of rows
def permute(idx: np.ndarray, plan, E: int, R: int):
    """Row of every (token, choice) assignment in the static per-rank buffers.

    Zero-copy placement ([MoonEP] para. 3): each assignment goes straight to its final
    row.  For assignment (t, j) with expert e, q = number of earlier tokens t' < t that
    chose e (token order within an expert).  A kept expert's rows start at its home
    offset: row = home(e)*C + expert_home_off[e] + q.  A streamed expert's assignment
    sits at stream position p = stream_off[e] + q; the rank u whose room range holds p
    receives it at row u*C + kept_rows[u] + (p - room_prefix[u]).

    Returns perm [T,k] int32 (row of each assignment) and src [R*C] int32 (token of
    each row).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    C = plan["C"]
    seen = [0] * E
    perm = np.full((T, k), -1, dtype=np.int32)
    src = np.full(R * C, -1, dtype=np.int32)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            q = seen[e]
            seen[e] += 1
            row = placement_row(e, q, plan, E, R)
            perm[t, j] = row
            src[row] = t
    return perm, src


def placement_row(e: int, q: int, plan, E: int, R: int) -> int:
    """Row of the q-th assignment (token order) of expert e under the plan: a kept
    expert's rows start at its home offset, home(e)*C + expert_home_off[e] + q; a streamed
    expert's assignment sits at stream position p = stream_off[e] + q and lands on the
    rank u whose room range [room_prefix[u], room_prefix[u+1]) holds p, at row
    u*C + kept_rows[u] + (p - room_prefix[u])."""
    C = plan["C"]
    B = E // R
    if plan["kept"][e]:
        return (e // B) * C + plan["expert_home_off"][e] + q
    rp = plan["room_prefix"]
    p = plan["stream_off"][e] + q
    u = 0
    while not (rp[u] <= p < rp[u + 1]):
        u += 1
    return u * C + plan["kept_rows"][u] + (p - rp[u])


def capacity_of(A: int, E: int, cf_num: int = 5, cf_den: int = 4) -> int:
    """Per-expert capacity of the fixed-capacity mode ([Hotspots] "Make expert capacity,
    overflow, and padding explicit"): ceil(assignments / experts * capacity factor), the
    factor an exact rational cf_num / cf_den (1.25 = 5/4 in the page's example)."""
    return -(-(A * cf_num) // (E * cf_den))


def dispatch_capacity(idx: np.ndarray, E: int, cap: int):
    """Fixed-capacity placement ([Hotspots] "Make expert capacity, overflow, and padding
    explicit"): every expert owns a static block of cap rows, rows [e*cap, (e+1)*cap), and
    the limit is applied to each expert independently.  The q-th assignment of expert e
    in token order (q = 0, 1, ...) is processed when q < cap and lands at row e*cap + q;
    the ones after it overflow and are dropped (perm = -1).  Rows of a block past the
    expert's processed count are padding (src = -1).  Which assignments the limit keeps is
    not on the page; token order is the plainest reading.  Overflow is counted from the
    raw demand before anything is excluded.

    Returns perm [T,k] int32 (row or -1), src [E*cap] int32 (token or -1), and the
    per-expert processed / overflow / padding counts as int64 arrays."""
    idx = np.asarray(idx)
    T, k = idx.shape
    seen = [0] * E
    perm = np.full((T, k), -1, dtype=np.int32)
    src = np.full(E * cap, -1, dtype=np.int32)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            q = seen[e]
            seen[e] += 1
            if q < cap:
                perm[t, j] = e * cap + q
                src[e * cap + q] = t
    demand = np.array(seen, dtype=np.int64)
    processed = np.minimum(demand, cap)
    return perm, src, dict(processed=processed, overflow=demand - processed,
                           padding=cap - processed)


def dispatch_padded(x: np.ndarray, src: np.ndarray) -> np.ndarray:
    """Rows of a fixed-capacity buffer: token src[r]'s row, zeros where src[r] = -1
    (padding)."""
    x = np.asarray(x)
    src = np.asarray(src)
    out = np.zeros((len(src), x.shape[1]), dtype=x.dtype)
    keep = src >= 0
    out[keep] = x[src[keep]]
    return out


def dispatch(x: np.ndarray, src: np.ndarray) -> np.ndarray:
    """Dispatch ([Primer] phase (b)): row r of the receive buffer is token src[r]'s row.
    A bitwise copy; each token lands once per chosen expert (O(top-k) volume)."""
    return np.asarray(x)[np.asarray(src)]


def prefetch(plan, W1, W3, W2, R: int, S: int):
    """Prefetch of redundant copies ([MoonEP] para. 3): pool slot u*S+s receives the
    home weights of replica_expert[u*S+s], bitwise, for all three projections.
    Returns dict slot -> (w1, w3, w2) for the filled slots."""
    out = {}
    for slot in range(R * S):
        e = plan["replica_expert"][slot]
        if e >= 0:
            out[slot] = (W1[e].copy(), W3[e].copy(), W2[e].copy())
    return out


# ------------------------------------------------------------------ expert FFN
def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), fp64."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(X, w1, w3, w2):
    """One SwiGLU expert on a block of rows, fp64 ([Primer] phase (c)):
    y = (silu(X w1^T) * (X w3^T)) w2^T with w1, w3 [F,d] and w2 [d,F]."""
    X = np.asarray(X, dtype=np.float64)
    g = X @ np.asarray(w1, dtype=np.float64).T
    u = X @ np.asarray(w3, dtype=np.float64).T
    h = silu(g) * u
    return h @ np.asarray(w2, dtype=np.float64).T


def weights_of(weight_ref: int, E: int, W1, W3, W2, pool):
    """Weights a group reads: the home tensor for weight_ref < E, else pool slot
    weight_ref - E."""
    if weight_ref < E:
        return W1[weight_ref], W3[weight_ref], W2[weight_ref]
    return pool[weight_ref - E]


def grouped_ffn(recv, plan, E: int, W1, W3, W2, pool, rows=None):
    """Grouped GEMM over the plan's groups ([Primer] phase (c)): every row of the
    receive buffer goes through the expert of the group holding it.  ``rows`` limits the
    evaluation to a subset (sampled parity); returns {row: y_row} then, else y [R*C,d]."""
    recv = np.asarray(recv)
    if rows is None:
        y = np.zeros((recv.shape[0], W2.shape[1]), dtype=np.float64)
        for u_groups in plan["groups"]:
            for (r0, n, e, ref) in u_groups:
                w1, w3, w2 = weights_of(ref, E, W1, W3, W2, pool)
                y[r0:r0 + n] = expert_ffn(recv[r0:r0 + n], w1, w3, w2)
        return y
    want = set(int(r) for r in rows)
    out = {}
    for u_groups in plan["groups"]:
        for (r0, n, e, ref) in u_groups:
            sel = [r for r in range(r0, r0 + n) if r in want]
            if not sel:
                continue
            w1, w3, w2 = weights_of(ref, E, W1, W3, W2, pool)
            ys = expert_ffn(recv[sel], w1, w3, w2)
            for r, yr in zip(sel, ys):
                out[r] = yr
    return out


# ------------------------------------------------------------------ combine
def combine(y, perm, gate, tokens=None):
    """Combine ([Primer] phase (d), the transpose of dispatch): token t's output is
    sum_j gate[t,j] * y[perm[t,j]], accumulated in j order in fp64.  ``y`` may be an
    array or a {row: vector} map (sampled parity); ``tokens`` limits the evaluation.
    An assignment dropped by the fixed-capacity mode (perm = -1) is left out of the sum;
    a token whose assignments were all dropped gets zeros."""
    perm = np.asarray(perm)
    gate = np.asarray(gate, dtype=np.float64)
    T, k = perm.shape
    toks = range(T) if tokens is None else tokens
    width = None
    out = {}
    for t in toks:
        acc = None
        for j in range(k):
            r = int(perm[t, j])
            if r < 0:
                continue
            v = gate[t, j] * np.asarray(y[r], dtype=np.float64)
            width = v.shape[0]
            acc = v if acc is None else acc + v
        out[int(t)] = acc
    for t in out:
        if out[t] is None:
            if width is None:
                width = (np.asarray(y).shape[1] if not isinstance(y, dict)
                         else len(next(iter(y.values()))))
            out[t] = np.zeros(width)
    if tokens is None:
        return np.stack([out[t] for t in range(T)]) if T else np.zeros((0, 0))
    return out


# ------------------------------------------------------------------ whole layer
def layer(logits, x, W1, W3, W2, k: int, R: int, S: int):
    """The whole path in the pages' order: route, measure, plan, prefetch, place rows,
    expert FFN, combine.  Small shapes only (loops are plain Python)."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx, gate, err = topk_route(logits, k)
    h = expert_histogram(idx, E, R)
    err |= h["err"]
    plan = plan_balanced(h["counts"], T, k, E, R, S)
    err |= plan["err"]
    pool = prefetch(plan, W1, W3, W2, R, S)
    perm, src = permute(idx, plan, E, R)
    recv = dispatch(x, src)
    y = grouped_ffn(recv, plan, E, W1, W3, W2, pool)
    out = combine(y, perm, gate)
    return dict(idx=idx, gate=gate, hist=h, plan=plan, pool=pool, perm=perm, src=src,
                recv=recv, y=y, out=out, err=err)



def layer_capacity(logits, x, W1, W3, W2, k: int, cf_num: int = 5, cf_den: int = 4):
    """The fixed-capacity (dropping) mode of the layer ([Hotspots] "Make expert capacity,
    overflow, and padding explicit"): route, measure the raw demand (the ledger is taken
    before any exclusion), place each expert's first cap assignments in its static
    block, run every expert over its whole block -- padding rows are zeros and cost the
    same work, the reserved work the page weighs against overflow -- and combine with the
    dropped assignments left out.  Small shapes only."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    A = T * k
    idx, gate, err = topk_route(logits, k)
    h = expert_histogram(idx, E, 1)
    err |= h["err"]
    cap = capacity_of(A, E, cf_num, cf_den)
    led = capacity_ledger(h["counts"], A, E, cf_num, cf_den)
    perm, src, rows = dispatch_capacity(idx, E, cap)
    recv = dispatch_padded(x, src)
    y = np.zeros((E * cap, np.asarray(W2).shape[1]))
    for e in range(E):
        y[e * cap:(e + 1) * cap] = expert_ffn(recv[e * cap:(e + 1) * cap], W1[e], W3[e], W2[e])
    out = combine(y, perm, gate)
    return dict(idx=idx, gate=gate, hist=h, cap=cap, ledger=led, rows=rows, perm=perm, src=src,
                recv=recv, y=y, out=out, err=err)


# ------------------------------------------------- expert parallelism, one process per GPU
# [MoonEP] para. 2-3 and [Primer] phases (b), (d): with one rank per GPU, every rank routes
# its own tokens, all ranks compute the same equal-load plan from the router output of
# the whole job, dispatch sends each assignment's row to the rank the plan gives it, each
# rank runs the FFN on the rows it received, and combine brings every processed row back
# to its token's rank.  Reading: the job's token order is rank-major (rank u's local token
# t is token u*T + t) and every rank holds the same number T of tokens, so the plan of the
# job is the plan of the concatenated batch with R = W ranks.

def ep_local_counts(idx_local, E: int):
    """Demand of one rank's own tokens: counts[e] = number of its assignments naming e
    (in-range ids only), and its validation bits."""
    idx_local = np.asarray(idx_local)
    counts = np.zeros(E, dtype=np.int64)
    for row in idx_local:
        for v in row:
            if 0 <= int(v) < E:
                counts[int(v)] += 1
    return counts, validate_trace(idx_local, E)


def ep_rank_base(counts_all, me: int):
    """Assignments of each expert made by lower ranks' tokens: with rank-major token
    order they come before rank me's in every expert's token order, so rank me's q of an
    assignment is q_base[e] = sum_{r < me} counts_all[r][e] plus its local rank."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    return counts_all[:me].sum(axis=0) if me > 0 else np.zeros(counts_all.shape[1], np.int64)


def ep_permute(idx_local, q_base, plan, E: int, R: int):
    """Job-wide row of each of one rank's assignments: the placement rule of permute()
    with q = q_base[e] + number of this rank's earlier tokens that chose e.  Row r lives
    on rank r // C at local row r % C.  Returns perm [T,k] int32."""
    idx_local = np.asarray(idx_local)
    T, k = idx_local.shape
    seen = [int(v) for v in q_base]
    perm = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        for j in range(k):
            e = int(idx_local[t, j])
            perm[t, j] = placement_row(e, seen[e], plan, E, R)
            seen[e] += 1
    return perm


def ep_layer(logits_shards, x_shards, W1, W3, W2, k: int, S: int):
    """The layer as W processes run it, one per GPU, rank u holding logits_shards[u] and
    x_shards[u] (T tokens each) and the home experts [u*B, (u+1)*B):
      1. route locally; count local demand; exchange the counts and error bits;
      2. every rank: job counts = sum over ranks, the same plan (R = W, T_job = W*T);
      3. prefetch: rank u's slots copy their experts' weights from the home ranks;
      4. dispatch: each assignment's row goes to rank perm // C, local row perm % C;
      5. every rank runs the grouped FFN on its own C rows and groups;
      6. combine: out[t] = sum_j gate[t,j] * y_{perm // C}[perm % C], in j order.
    Returns dict(ranks=[per-rank dict(idx, gate, perm, recv, y, out)], plan, counts_all,
    err)."""
    W = len(logits_shards)
    E = np.asarray(logits_shards[0]).shape[1]
    T = np.asarray(logits_shards[0]).shape[0]
    ranks = []
    err = 0
    for u in range(W):
        idx, gate, e_route = topk_route(np.asarray(logits_shards[u], dtype=np.float32), k)
        c, e_val = ep_local_counts(idx, E)
        ranks.append(dict(idx=idx, gate=gate, counts=c))
        err |= e_route | e_val
    counts_all = np.stack([r["counts"] for r in ranks])
    counts = counts_all.sum(axis=0)
    plan = plan_balanced(counts, W * T, k, E, W, S)
    err |= plan["err"]
    C = plan["C"]
    pool = prefetch(plan, W1, W3, W2, W, S)
    d = np.asarray(x_shards[0]).shape[1]
    recv = [np.zeros((C, d), dtype=np.asarray(x_shards[0]).dtype) for _ in range(W)]
    for u in range(W):
        perm = ep_permute(ranks[u]["idx"], ep_rank_base(counts_all, u), plan, E, W)
        ranks[u]["perm"] = perm
        xs = np.asarray(x_shards[u])
        for t in range(T):
            for j in range(k):
                r = int(perm[t, j])
                recv[r // C][r % C] = xs[t]
    for u in range(W):
        y = np.zeros((C, np.asarray(W2).shape[1]), dtype=np.float64)
        for (r0, n, e, ref) in plan["groups"][u]:
            w1, w3, w2 = weights_of(ref, E, W1, W3, W2, pool)
            y[r0 - u * C:r0 - u * C + n] = expert_ffn(recv[u][r0 - u * C:r0 - u * C + n], w1, w3, w2)
        ranks[u]["recv"] = recv[u]
        ranks[u]["y"] = y
    for u in range(W):
        perm, gate = ranks[u]["perm"], ranks[u]["gate"]
        out = np.zeros((T, np.asarray(W2).shape[1]))
        for t in range(T):
            for j in range(k):
                r = int(perm[t, j])
                out[t] += float(gate[t, j]) * ranks[r // C]["y"][r % C]
        ranks[u]["out"] = out
    return dict(ranks=ranks, plan=plan, pool=pool, counts_all=counts_all, err=err)


# ------------------------------------------------------------------ backward pass
# [MoonEP] para. 3: the duplicated experts' "gradients get reduced back home during the
# backward pass".  The pages give no formulas; these are the chain rule through the
# forward above, with the reading that top-k selection passes no gradient to the
# experts it did not choose (it is piecewise constant in the logits).

def silu_grad(z):
    """d silu / dz = sigmoid(z) * (1 + z * (1 - sigmoid(z))), fp64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def combine_backward(dout, y, perm, gate):
    """Backward of combine: out[t] = sum_j gate[t,j] y[perm[t,j]], so
    dy[perm[t,j]] = gate[t,j] dout[t] and dgate[t,j] = <dout[t], y[perm[t,j]]>."""
    dout = np.asarray(dout, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    perm = np.asarray(perm)
    gate = np.asarray(gate, dtype=np.float64)
    T, k = perm.shape
    dy = np.zeros_like(y)
    dgate = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            r = int(perm[t, j])
            dy[r] = gate[t, j] * dout[t]
            dgate[t, j] = float(dout[t] @ y[r])
    return dy, dgate


def expert_ffn_backward(X, w1, w3, w2, dy):
    """Backward of one SwiGLU expert on a block of rows, fp64.  Forward: g = X w1^T,
    u = X w3^T, h = silu(g) u, y = h w2^T.  Returns the row gradient dX and the weight
    gradients of this block, plus the intermediates dh, dg, du."""
    X = np.asarray(X, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w3 = np.asarray(w3, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    g = X @ w1.T
    u = X @ w3.T
    sg = silu(g)
    h = sg * u
    dh = dy @ w2              # [n,F]
    dw2 = dy.T @ h            # [d,F]
    du = dh * sg
    dg = dh * u * silu_grad(g)
    dX = dg @ w1 + du @ w3    # [n,d]
    dw1 = dg.T @ X            # [F,d]
    dw3 = du.T @ X
    return dict(dX=dX, dw1=dw1, dw3=dw3, dw2=dw2, dh=dh, dg=dg, du=du, h=h)


def grouped_ffn_backward(recv, dy, plan, E: int, W1, W3, W2, pool):
    """Backward of the grouped FFN: every group's rows through its expert's backward.
    A replica slot holds its expert's weights bitwise, and the gradient of every group --
    home or replica -- is added to its expert's home gradient ([MoonEP] para. 3: replica
    gradients are reduced back home).  Returns dX rows [R*C,d], dW1, dW3 [E,F,d], dW2
    [E,d,F] and the per-row intermediates dh, dg, du [R*C,F]."""
    recv = np.asarray(recv, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    rows, d = recv.shape
    F = W1.shape[1]
    dX = np.zeros((rows, d))
    dh = np.zeros((rows, F))
    dg = np.zeros((rows, F))
    du = np.zeros((rows, F))
    dW1 = np.zeros((E, F, d))
    dW3 = np.zeros((E, F, d))
    dW2 = np.zeros((E, d, F))
    for u_groups in plan["groups"]:
        for (r0, n, e, ref) in u_groups:
            w1, w3, w2 = weights_of(ref, E, W1, W3, W2, pool)
            b = expert_ffn_backward(recv[r0:r0 + n], w1, w3, w2, dy[r0:r0 + n])
            dX[r0:r0 + n] = b["dX"]
            dh[r0:r0 + n] = b["dh"]
            dg[r0:r0 + n] = b["dg"]
            du[r0:r0 + n] = b["du"]
            dW1[e] += b["dw1"]
            dW3[e] += b["dw3"]
            dW2[e] += b["dw2"]
    return dict(dX=dX, dW1=dW1, dW3=dW3, dW2=dW2, dh=dh, dg=dg, du=du)


def dispatch_backward(dX, perm):
    """Backward of dispatch (recv[perm[t,j]] = x[t]): dx[t] = sum_j dX[perm[t,j]], in j
    order."""
    dX = np.asarray(dX, dtype=np.float64)
    perm = np.asarray(perm)
    T, k = perm.shape
    dx = np.zeros((T, dX.shape[1]))
    for t in range(T):
        for j in range(k):
            dx[t] += dX[int(perm[t, j])]
    return dx


def topk_backward(gate, dgate, idx, E: int):
    """Backward of the gates: gate = softmax over the chosen logits, so
    dlogit[t, idx[t,j]] = gate[t,j] (dgate[t,j] - sum_i gate[t,i] dgate[t,i]); experts not
    chosen get 0 (the selection itself passes no gradient)."""
    gate = np.asarray(gate, dtype=np.float64)
    dgate = np.asarray(dgate, dtype=np.float64)
    idx = np.asarray(idx)
    T, k = idx.shape
    dl = np.zeros((T, E))
    for t in range(T):
        s = float(gate[t] @ dgate[t])
        for j in range(k):
            dl[t, int(idx[t, j])] = gate[t, j] * (dgate[t, j] - s)
    return dl


def layer_backward(fwd, dout, W1, W3, W2, E: int):
    """The backward of layer() given its outputs ``fwd`` and dout = dLoss/dout [T,d]:
    combine, expert FFN (replica gradients reduced home), dispatch, gates.  Returns dx
    [T,d], dlogits [T,E], dW1, dW3, dW2 and the intermediates."""
    dy, dgate = combine_backward(dout, fwd["y"], fwd["perm"], fwd["gate"])
    g = grouped_ffn_backward(fwd["recv"], dy, fwd["plan"], E, W1, W3, W2, fwd["pool"])
    dx = dispatch_backward(g["dX"], fwd["perm"])
    dlogits = topk_backward(fwd["gate"], dgate, fwd["idx"], E)
    return dict(dx=dx, dlogits=dlogits, dW1=g["dW1"], dW3=g["dW3"], dW2=g["dW2"], dy=dy,
                dgate=dgate, dX_rows=g["dX"], dh=g["dh"], dg=g["dg"], du=g["du"])


def ep_layer_backward(ep, douts, W1, W3, W2, E: int, S: int):
    """The backward of ep_layer() as the W processes run it, rank u holding douts[u]
    ([MoonEP] para. 3: the duplicated experts' gradients are reduced back home):
      1. combine backward across ranks: for each of rank u's assignments (t, j) with row
         r on rank v = r // C: v's dy[r % C] = gate[t,j] dout[t]; dgate[t,j] =
         <dout[t], y_v[r % C]>;
      2. every rank v: each of its groups through its expert's backward on v's own rows
         (dX rows); a home group's weight gradient goes to v's partial of that home
         expert, a replica group's to v's partial of that pool slot;
      3. reduction back home: expert e's gradient, on rank e // B, is its home partial plus
         the partial of every slot (v, s) that held a copy of e, in (v, s) order;
      4. dispatch backward across ranks: dx[t] = sum_j dX_v[r % C], in j order;
      5. the gates' backward, local.
    Returns dict(ranks=[dict(dy, dgate, dX_rows, dx, dlogits)], dW1, dW3, dW2 [E,...])."""
    ranks = ep["ranks"]
    plan = ep["plan"]
    W = len(ranks)
    C = plan["C"]
    B = E // W
    d = np.asarray(W1).shape[2]
    F = np.asarray(W1).shape[1]
    dys = [np.zeros((C, d)) for _ in range(W)]
    out = [dict() for _ in range(W)]
    for u, r in enumerate(ranks):
        dout = np.asarray(douts[u], dtype=np.float64)
        perm, gate = r["perm"], np.asarray(r["gate"], dtype=np.float64)
        T, k = perm.shape
        dgate = np.zeros((T, k))
        for t in range(T):
            for j in range(k):
                row = int(perm[t, j])
                v = row // C
                dys[v][row % C] = gate[t, j] * dout[t]
                dgate[t, j] = float(dout[t] @ np.asarray(ranks[v]["y"], dtype=np.float64)[row % C])
        out[u]["dgate"] = dgate
    parts = []
    for v in range(W):
        recv = np.asarray(ranks[v]["recv"], dtype=np.float64)
        dX = np.zeros((C, d))
        part1 = np.zeros((B + S, F, d))
        part3 = np.zeros((B + S, F, d))
        part2 = np.zeros((B + S, d, F))
        for (r0, n, e, ref) in plan["groups"][v]:
            lo = r0 - v * C
            w1, w3, w2 = weights_of(ref, E, W1, W3, W2, ep["pool"])
            b = expert_ffn_backward(recv[lo:lo + n], w1, w3, w2, dys[v][lo:lo + n])
            dX[lo:lo + n] = b["dX"]
            slot = e - v * B if ref < E else B + (ref - E - v * S)
            part1[slot] += b["dw1"]
            part3[slot] += b["dw3"]
            part2[slot] += b["dw2"]
        out[v]["dy"] = dys[v]
        out[v]["dX_rows"] = dX
        parts.append((part1, part3, part2))
    dW1 = np.zeros((E, F, d))
    dW3 = np.zeros((E, F, d))
    dW2 = np.zeros((E, d, F))
    for e in range(E):
        home = e // B
        acc = [parts[home][i][e - home * B].copy() for i in range(3)]
        for v in range(W):
            for s in range(S):
                if plan["replica_expert"][v * S + s] == e:
                    for i in range(3):
                        acc[i] += parts[v][i][B + s]
        dW1[e], dW3[e], dW2[e] = acc
    for u, r in enumerate(ranks):
        perm = r["perm"]
        T, k = perm.shape
        dx = np.zeros((T, d))
        for t in range(T):
            for j in range(k):
                row = int(perm[t, j])
                dx[t] += out[row // C]["dX_rows"][row % C]
        out[u]["dx"] = dx
        out[u]["dlogits"] = topk_backward(r["gate"], out[u]["dgate"], r["idx"], E)
    return dict(ranks=out, dW1=dW1, dW3=dW3, dW2=dW2)
