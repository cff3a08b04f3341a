"""Plain fp64 CPU oracle for SQuad-Attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or executes this module: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and ``--impl
reference``) may use it. It shares no code with the CUDA library; both sides are fed from the seeded
generator in ``sub_quadratic_two_squad_b200/inputs.py``, which holds no attention arithmetic.

Sources ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video Generation", as printed on
the paperpeel.com page, the agihunt.info digest, the romaanj.github.io review and the gist.science
summary):

* Full softmax self-attention softmax(Q K^T / sqrt(d)) V per head -- paper §3.1 (eq. 5).
* SQuad-Attention is a sequence of two plain softmax attentions, the second fed by the first; the
  passes are joined by re-indexing alone: each takes the axis it attends over as its sequence and
  merges the remaining index into the batch of heads -- agihunt.info digest, the paragraph that
  defines the operator; paper appendix "Cost of the two passes" and "Analyzing the results".
* Local pass: each token attends inside its window; the window covers every frame and an hw x ww
  block of space (e.g. 21x2x4 = 168 tokens at n = 18480) -- agihunt.info digest, the paragraph on the
  window size; review, "Method".
* Global pass: tokens at the same position (slot) inside their windows attend across all windows, and
  the local output is its value stream -- paper appendix "Reachability" (two-hop path (c',j') ->
  (c',j) -> (c,j)); gist.science summary, item "Composição".
* Order: local->global is the paper's default, global->local the ablated reverse; for G->L the
  effective weight is beta_{j->j'}^{c} alpha_{c->c'}^{j'} -- paper appendix "On the ordering".
* Cost: 4hd(n w + n^2 / w) for the two passes and 4hdn^2 for full attention -- paper appendix
  "Conformance to the theoretical curves is quantitative".

Readings where the pages are silent (equations 7-9 were lost in extraction):

* Pass 2 takes the same Q and K, rearranged to the slot view; its values are the pass-1 output.
* Both passes use the eq. 5 scale 1/sqrt(d) unless the caller passes another.
* Tokens are flattened (t, y, x) row-major: token = (t*H + y)*W + x. Window c = (wy, wx) runs
  row-major over (H/hw, W/ww); slot j = (t, dy, dx) runs row-major over (tw, hw, ww). The result does
  not depend on these orders (softmax sums are permutation invariant; outputs go back to token order).
* The backward pass is the chain rule through both passes; the pages do not print it.
* Grids the window does not divide (paper appendix, "Conformance to the theoretical curves is
  quantitative": such grids are reflect-padded, and at each resolution the window is chosen anew,
  spanning all frames, with a height-to-width split set by the grid's aspect ratio). Readings: reflect padding
  (the edge token is not repeated) at the bottom of H and the right of W in every frame, up to the next
  multiple of the window; both passes run on the padded grid and the output is cropped back, so the
  gradient of an input token sums over its padded copies. The solver takes, among windows with
  w_t = T and for each w_h the w_w whose ratio w_h:w_w is closest to H:W (log ratio), the one with the
  least cost n'm + n'^2/m on the padded count n'.

* More than two passes (the paper names composing more passes as open, §5 "Limitations and future
  work", and defines none): nested windows, each spatial axis factored into k levels, pass p
  attending along level p's digits with the others fixed (pass 1 also along the frames); k = 2 is
  SQuad, k = 1 full attention. See the k-pass section below.

Every array here is float64. Pins: tests/test_oracle_pins.py and tests/test_oracle_kpass.py.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------------------------
# Re-indexing (the "local" and "global" token views)
# ----------------------------------------------------------------------------------------------

def window_partition(T: int, H: int, W: int, tw: int, hw: int, ww: int) -> np.ndarray:
    """Token index of slot j inside window c, as an int array [N_w, w].

    Row c lists the w = tw*hw*ww tokens of window c (the local pass attends along a row); column j
    lists the N_w tokens that occupy slot j in every window (the global pass attends along a column).
    """
    if tw != T:
        raise ValueError("the window covers every frame: tw must equal T")
    if H % hw or W % ww:
        raise ValueError("window must tile the H x W grid exactly")
    nwy, nwx = H // hw, W // ww
    table = np.empty((nwy * nwx, tw * hw * ww), dtype=np.int64)
    for wy in range(nwy):
        for wx in range(nwx):
            c = wy * nwx + wx
            for t in range(tw):
                for dy in range(hw):
                    for dx in range(ww):
                        j = (t * hw + dy) * ww + dx
                        y = wy * hw + dy
                        x = wx * ww + dx
                        table[c, j] = (t * H + y) * W + x
    return table


# ----------------------------------------------------------------------------------------------
# One softmax attention over a batch of sequences (eq. 5)
# ----------------------------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """softmax(q k^T * scale) v over the last-but-one axis; returns (out, lse).

    q: [..., s, d], k: [..., s, d], v: [..., s, dv]. lse is the natural-log log-sum-exp of the scaled
    scores per query row, [..., s]. The softmax subtracts the row maximum (exact in real arithmetic).
    """
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * scale
    m = s.max(axis=-1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=-1, keepdims=True)
    out = np.matmul(p / l, v)
    lse = (m + np.log(l))[..., 0]
    return out, lse


def softmax_attention_bwd(q, k, v, dout, scale: float):
    """Gradients (dq, dk, dv) of <dout, softmax(q k^T * scale) v> by the chain rule.

    P = softmax(S), S = scale q k^T, out = P v:
      dv = P^T dout;  dP = dout v^T;  dS = P * (dP - rowsum(dP * P));  dq = scale dS k;  dk = scale dS^T q.
    """
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    dv = np.matmul(np.swapaxes(p, -1, -2), dout)
    dp = np.matmul(dout, np.swapaxes(v, -1, -2))
    ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))
    dq = np.matmul(ds, k) * scale
    dk = np.matmul(np.swapaxes(ds, -1, -2), q) * scale
    return dq, dk, dv


# ----------------------------------------------------------------------------------------------
# The two passes
# ----------------------------------------------------------------------------------------------

def _scale(d: int, scale):
    return 1.0 / np.sqrt(d) if scale is None else float(scale)


def _pass(Q, K, V, groups: np.ndarray, scale: float):
    """Attention inside every group of tokens (a row of ``groups`` is one sequence), per (b, head).

    Q, K: [B, h, n, d]; V: [B, h, n, dv]; groups: [G, s] token indices. Returns (out [B,h,n,dv],
    lse [B,h,n]). Heads are independent, so they are processed one at a time to bound memory.
    """
    B, h, n, _ = Q.shape
    out = np.empty(V.shape, dtype=np.float64)
    lse = np.empty((B, h, n), dtype=np.float64)
    for b in range(B):
        for hh in range(h):
            qg = Q[b, hh][groups]          # [G, s, d]
            kg = K[b, hh][groups]
            vg = V[b, hh][groups]          # [G, s, dv]
            o, l = softmax_attention(qg, kg, vg, scale)
            out[b, hh][groups] = o
            lse[b, hh][groups] = l
    return out, lse


def local_pass(Q, K, V, grid, window, scale=None):
    """Attn_L: full softmax attention inside each window of tw x hw x ww tokens (tw = T)."""
    table = window_partition(*grid, *window)
    return _pass(_f64(Q), _f64(K), _f64(V), table, _scale(Q.shape[-1], scale))


def global_pass(Q, K, V, grid, window, scale=None):
    """Attn_G: for every slot j, the tokens at slot j of all n/w windows attend to one another."""
    table = window_partition(*grid, *window)
    return _pass(_f64(Q), _f64(K), _f64(V), np.ascontiguousarray(table.T), _scale(Q.shape[-1], scale))


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------------------------
# Grids the window does not divide: reflect padding, cropping, and the window solver
# ----------------------------------------------------------------------------------------------

def padded_grid(grid, window):
    """(T, H', W'): H and W rounded up to multiples of the window's hw and ww."""
    T, H, W = grid
    _, hw, ww = window
    return T, -(-H // hw) * hw, -(-W // ww) * ww


def divides(grid, window):
    return tuple(padded_grid(grid, window)) == tuple(grid)


def reflect_pad_tokens(X, grid, window):
    """[B, h, n, d] -> [B, h, n', d]: each frame reflect-padded at the bottom and right ends."""
    T, H, W = grid
    _, Hp, Wp = padded_grid(grid, window)
    if Hp - H > H - 1 or Wp - W > W - 1:
        raise ValueError("reflect padding needs a pad shorter than the extent")
    B, h, n, d = X.shape
    x = np.asarray(X).reshape(B, h, T, H, W, d)
    x = np.pad(x, ((0, 0), (0, 0), (0, 0), (0, Hp - H), (0, Wp - W), (0, 0)), mode="reflect")
    return x.reshape(B, h, T * Hp * Wp, d)


def crop_tokens(X, grid, window):
    """[B, h, n', d] -> [B, h, n, d]: the tokens of the original grid."""
    T, H, W = grid
    _, Hp, Wp = padded_grid(grid, window)
    B, h, _, d = X.shape
    return np.ascontiguousarray(np.asarray(X).reshape(B, h, T, Hp, Wp, d)[:, :, :, :H, :W]).reshape(B, h, T * H * W, d)


def fold_reflect_grad(G, grid, window):
    """Adjoint of reflect_pad_tokens: the gradient on the padded grid summed onto the source tokens."""
    T, H, W = grid
    _, Hp, Wp = padded_grid(grid, window)
    B, h, _, d = G.shape
    g = np.asarray(G).reshape(B, h, T, Hp, Wp, d)
    src_y = np.array([i if i < H else 2 * (H - 1) - i for i in range(Hp)])
    src_x = np.array([i if i < W else 2 * (W - 1) - i for i in range(Wp)])
    out = np.zeros((B, h, T, H, W, d), dtype=np.float64)
    for yp in range(Hp):
        for xp in range(Wp):
            out[:, :, :, src_y[yp], src_x[xp]] += g[:, :, :, yp, xp]
    return out.reshape(B, h, T * H * W, d)


def _aspect_ww(hw: int, H: int, W: int) -> int:
    """The ww whose ratio hw:ww is closest to H:W (in log ratio; the lower one on a tie)."""
    lo = max(1, int(np.floor(hw * W / H)))
    cands = (lo, lo + 1)
    return min(cands, key=lambda ww: (abs(np.log(hw / ww) - np.log(H / W)), ww))


def window_solve(T: int, H: int, W: int):
    """The window (T, hw, ww) for a T x H x W grid: w_t = T, ww following the aspect ratio for each hw,
    and the hw whose padded cost n'm + n'^2/m (m = T hw ww, n' = the reflect-padded token count) is
    least (paper appendix "What is measured" for the rule; "Conformance to the theoretical curves is
    quantitative" for scoring the cost of the window actually used)."""
    best = None
    for hw in range(1, H + 1):
        ww = _aspect_ww(hw, H, W)
        if ww > W:
            continue
        _, Hp, Wp = padded_grid((T, H, W), (T, hw, ww))
        if Hp - H > H - 1 or Wp - W > W - 1:
            continue
        n_p, m = T * Hp * Wp, T * hw * ww
        cost = n_p * m + n_p * n_p / m
        if best is None or cost < best[0]:
            best = (cost, hw, ww)
    return T, best[1], best[2]


LOCAL_THEN_GLOBAL = "local_then_global"
GLOBAL_THEN_LOCAL = "global_then_local"
# Single-pass variants: each pass alone, as the paper ablates them (SQuad paper §4.4, "The need for and
# the order of the two passes").
LOCAL_ONLY = "local_only"
GLOBAL_ONLY = "global_only"
SINGLE_PASS = (LOCAL_ONLY, GLOBAL_ONLY)


def squad_attn_fwd(Q, K, V, grid, window, order=LOCAL_THEN_GLOBAL, scale=None, return_aux=False):
    """SQuad-Attention forward: the two passes composed, pass 2 taking pass 1's output as values.

    grid = (T, H, W); window = (tw, hw, ww). Q, K: [B, h, n, d], V: [B, h, n, dv] with n = T*H*W.
    With return_aux, also returns dict(o1=..., lse1=..., lse2=...) (pass-1 output and both passes'
    log-sum-exp).
    """
    if not divides(grid, window):
        # reflect-pad, run on the padded grid, crop the output (aux arrays stay on the padded grid)
        pg = padded_grid(grid, window)
        res = squad_attn_fwd(*(reflect_pad_tokens(_f64(X), grid, window) for X in (Q, K, V)), pg, window, order,
                             scale, return_aux)
        o = res[0] if return_aux else res
        o = crop_tokens(o, grid, window)
        return (o, res[1]) if return_aux else o
    if order in SINGLE_PASS:
        o, lse = (local_pass if order == LOCAL_ONLY else global_pass)(Q, K, V, grid, window, scale)
        return (o, dict(lse1=lse)) if return_aux else o
    if order not in (LOCAL_THEN_GLOBAL, GLOBAL_THEN_LOCAL):
        raise ValueError(order)
    first, second = (local_pass, global_pass) if order == LOCAL_THEN_GLOBAL else (global_pass, local_pass)
    o1, lse1 = first(Q, K, V, grid, window, scale)
    o, lse2 = second(Q, K, o1, grid, window, scale)
    if return_aux:
        return o, dict(o1=o1, lse1=lse1, lse2=lse2)
    return o


def squad_attn_bwd(Q, K, V, dO, grid, window, order=LOCAL_THEN_GLOBAL, scale=None):
    """Gradients (dQ, dK, dV) of <dO, squad_attn_fwd(Q, K, V)>.

    Reverse of the two passes: pass 2's backward (values = pass-1 output) gives its share of dQ and dK
    and the gradient dO1 of the pass-1 output; pass 1's backward with upstream dO1 gives the rest of dQ
    and dK, and dV. Q and K are used by both passes, so each receives the sum of two terms.
    """
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    if not divides(grid, window):
        # the padded method: pad (reflect), both passes, crop; so dO is zero on the padded tokens and
        # each input token's gradient sums over its padded copies
        pg = padded_grid(grid, window)
        B, h, _, d = dO.shape
        do_p = np.zeros((B, h, pg[0] * pg[1] * pg[2], d))
        do_p.reshape(B, h, pg[0], pg[1], pg[2], d)[:, :, :, :grid[1], :grid[2]] = dO.reshape(B, h, *grid, d)
        grads = squad_attn_bwd(*(reflect_pad_tokens(X, grid, window) for X in (Q, K, V)), do_p, pg, window, order,
                               scale)
        return tuple(fold_reflect_grad(G, grid, window) for G in grads)
    sc = _scale(Q.shape[-1], scale)
    table = window_partition(*grid, *window)
    local_groups, global_groups = table, np.ascontiguousarray(table.T)
    if order in SINGLE_PASS:
        # one softmax attention per sequence of the pass
        g = local_groups if order == LOCAL_ONLY else global_groups
        dQ, dK, dV = np.empty_like(Q), np.empty_like(K), np.empty_like(V)
        for b in range(Q.shape[0]):
            for hh in range(Q.shape[1]):
                dq, dk, dv = softmax_attention_bwd(Q[b, hh][g], K[b, hh][g], V[b, hh][g], dO[b, hh][g], sc)
                dQ[b, hh][g], dK[b, hh][g], dV[b, hh][g] = dq, dk, dv
        return dQ, dK, dV
    if order not in (LOCAL_THEN_GLOBAL, GLOBAL_THEN_LOCAL):
        raise ValueError(order)
    g1, g2 = (local_groups, global_groups) if order == LOCAL_THEN_GLOBAL else (global_groups, local_groups)
    o1, _ = _pass(Q, K, V, g1, sc)

    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.empty_like(V)
    B, h = Q.shape[:2]
    for b in range(B):
        for hh in range(h):
            q, k, v, do, x1 = Q[b, hh], K[b, hh], V[b, hh], dO[b, hh], o1[b, hh]
            dq2, dk2, do1 = softmax_attention_bwd(q[g2], k[g2], x1[g2], do[g2], sc)
            d_o1 = np.empty_like(x1)
            d_o1[g2] = do1
            dq1, dk1, dv1 = softmax_attention_bwd(q[g1], k[g1], v[g1], d_o1[g1], sc)
            dq = np.zeros_like(q)
            dk = np.zeros_like(k)
            dq[g2] += dq2
            dk[g2] += dk2
            dq[g1] += dq1
            dk[g1] += dk1
            dQ[b, hh] = dq
            dK[b, hh] = dk
            dV[b, hh][g1] = dv1
    return dQ, dK, dV


# ----------------------------------------------------------------------------------------------
# Full attention, the composed weight matrix, and the cost model
# ----------------------------------------------------------------------------------------------

def full_attn_fwd(Q, K, V, scale=None, rows=None):
    """softmax(Q K^T * scale) V over all n tokens per head (eq. 5); optionally only query ``rows``.

    Returns (out [B,h,r,dv], lse [B,h,r]) with r = n or len(rows).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    sc = _scale(Q.shape[-1], scale)
    if rows is not None:
        Q = Q[:, :, np.asarray(rows), :]
    B, h = Q.shape[:2]
    out = np.empty(Q.shape[:3] + (V.shape[-1],))
    lse = np.empty(Q.shape[:3])
    for b in range(B):
        for hh in range(h):
            out[b, hh], lse[b, hh] = softmax_attention(Q[b, hh], K[b, hh], V[b, hh], sc)
    return out, lse


def composed_matrix(Q, K, grid, window, order=LOCAL_THEN_GLOBAL, scale=None):
    """The n x n matrix M with squad_attn_fwd(Q, K, V) = M V, per (b, head).

    Obtained by pushing the n one-hot value vectors through both passes (V = identity, dv = n). Entry
    M[u, v] is the effective weight gamma from source token v to target token u (paper appendix
    "Reachability": the local weight times the global weight along the two-hop path).
    """
    B, h, n, _ = Q.shape
    eye = np.broadcast_to(np.eye(n), (B, h, n, n))
    return squad_attn_fwd(Q, K, eye, grid, window, order, scale)


def squad_flops(B: int, h: int, d: int, n: int, w: int) -> float:
    """4 B h d (n w + n^2 / w): QK^T and PV of the local pass (n/w windows of w tokens) plus those of
    the global pass (w slots of n/w tokens); each GEMM of an s-token sequence costs 2 s^2 d FLOPs."""
    return 4.0 * B * h * d * (n * w + n * n / w)


def full_flops(B: int, h: int, d: int, n: int) -> float:
    """4 B h d n^2: QK^T and PV of full attention."""
    return 4.0 * B * h * d * n * n


# ----------------------------------------------------------------------------------------------
# More than two composed passes: nested windows
# ----------------------------------------------------------------------------------------------
# The paper names composing more than two passes as an open direction (§5 "Limitations and future
# work"; review, "Sparks") and defines no partition for a third pass. The reading taken here is the
# plainest generalisation of the two passes, nested windows:
#
# * each spatial axis is factored into k levels, H = h_1 h_2 ... h_k and W = w_1 w_2 ... w_k, and a
#   token's row and column are mixed-radix numbers with level 1 least significant:
#   y = a_1 + h_1 (a_2 + h_2 (a_3 + ...)), x = b_1 + w_1 (b_2 + w_2 (b_3 + ...)), 0 <= a_p < h_p,
#   0 <= b_p < w_p;
# * pass p attends among the tokens that agree on every digit except (a_p, b_p); pass 1 also spans
#   all frames t (the window of the two-pass method covers every frame), the other passes keep t;
# * every pass takes the same Q and K; its values are the previous pass's output (v for the first).
#
# With k = 2 this is SQuad with window (T, h_1, w_1): pass 1 is the local pass (inside a window),
# pass 2 the global pass (one slot across the h_2 x w_2 windows). With k = 1 it is full attention.
# "forward" runs level 1 first (the analogue of local->global), "reverse" level k first.

KPASS_FORWARD = "forward"
KPASS_REVERSE = "reverse"


def _check_levels(grid, levels):
    T, H, W = grid
    levels = [(int(a), int(b)) for a, b in levels]
    if not levels or any(a < 1 or b < 1 for a, b in levels):
        raise ValueError("levels: k >= 1 pairs (h_p, w_p) of positive integers")
    if int(np.prod([a for a, _ in levels])) != H or int(np.prod([b for _, b in levels])) != W:
        raise ValueError("the levels must factor the grid: prod h_p = H and prod w_p = W")
    return levels


def level_groups(grid, levels, p: int) -> np.ndarray:
    """Token indices of the sequences of pass p (0-based level), as an int array [G, s].

    A row lists the tokens that share every digit except level p's (and, for p = 0, the frame), in a
    fixed order; the rows partition the n tokens.
    """
    T, H, W = grid
    levels = _check_levels(grid, levels)
    tok = np.arange(T * H * W, dtype=np.int64)
    t, y, x = tok // (H * W), (tok // W) % H, tok % W
    a, b = [], []
    for hp, wp in levels:
        a.append(y % hp)
        b.append(x % wp)
        y, x = y // hp, x // wp
    hp, wp = levels[p]
    member = a[p] * wp + b[p]
    size = hp * wp
    if p == 0:
        member = t * size + member
        size *= T
    key = np.zeros_like(tok)
    for q, (hq, wq) in enumerate(levels):
        if q != p:
            key = key * (hq * wq) + a[q] * wq + b[q]
    if p != 0:
        key = key * T + t
    order = np.lexsort((member, key))
    return tok[order].reshape(-1, size)


def _kpass_levels_in_order(levels, order):
    if order not in (KPASS_FORWARD, KPASS_REVERSE):
        raise ValueError(order)
    idx = list(range(len(levels)))
    return idx if order == KPASS_FORWARD else idx[::-1]


def kpass_fwd(Q, K, V, grid, levels, order=KPASS_FORWARD, scale=None, return_aux=False):
    """k nested-window passes composed, each taking the previous one's output as values.

    grid = (T, H, W); levels = [(h_1, w_1), ..., (h_k, w_k)]. With return_aux, also returns the inputs
    of every executed pass's values and each pass's log-sum-exp (lists in execution order).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    sc = _scale(Q.shape[-1], scale)
    values, lses = [], []
    x = V
    for p in _kpass_levels_in_order(levels, order):
        values.append(x)
        x, lse = _pass(Q, K, x, level_groups(grid, levels, p), sc)
        lses.append(lse)
    if return_aux:
        return x, dict(values=values, lse=lses)
    return x


def kpass_bwd(Q, K, V, dO, grid, levels, order=KPASS_FORWARD, scale=None):
    """Gradients (dQ, dK, dV) of <dO, kpass_fwd(Q, K, V)>: the passes' backward in reverse execution
    order, each passing the gradient of its values on to the pass before; dQ and dK sum every pass's
    share."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    sc = _scale(Q.shape[-1], scale)
    seq = _kpass_levels_in_order(levels, order)
    _, aux = kpass_fwd(Q, K, V, grid, levels, order, scale, return_aux=True)
    dQ, dK = np.zeros_like(Q), np.zeros_like(K)
    g = dO
    B, h = Q.shape[:2]
    for e in range(len(seq) - 1, -1, -1):
        groups = level_groups(grid, levels, seq[e])
        x = aux["values"][e]
        gv = np.empty_like(x)
        for b in range(B):
            for hh in range(h):
                dq, dk, dv = softmax_attention_bwd(Q[b, hh][groups], K[b, hh][groups], x[b, hh][groups],
                                                   g[b, hh][groups], sc)
                dQ[b, hh][groups] += dq
                dK[b, hh][groups] += dk
                gv[b, hh][groups] = dv
        g = gv
    return dQ, dK, g


def kpass_composed_matrix(Q, K, grid, levels, order=KPASS_FORWARD, scale=None):
    """The n x n matrix M with kpass_fwd(Q, K, V) = M V, per (b, head) (one-hot values)."""
    B, h, n, _ = Q.shape
    eye = np.broadcast_to(np.eye(n), (B, h, n, n))
    return kpass_fwd(Q, K, eye, grid, levels, order, scale)


def kpass_flops(B: int, h: int, d: int, grid, levels) -> float:
    """4 B h d n (m_1 + ... + m_k): pass p runs n/m_p sequences of m_p tokens (m_1 = T h_1 w_1,
    m_p = h_p w_p otherwise), each costing 4 m_p^2 d FLOPs for QK^T and PV."""
    T, H, W = grid
    levels = _check_levels(grid, levels)
    n = T * H * W
    m = [T * levels[0][0] * levels[0][1]] + [a * b for a, b in levels[1:]]
    return 4.0 * B * h * d * n * float(sum(m))
