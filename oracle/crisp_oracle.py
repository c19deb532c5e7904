"""CRISP sparse-prefill oracle — plain, slow, fp64, CPU.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module; the library itself never calls it and has no CPU fallback.

Every function restates one step of the method as the pages define it, in fp64 numpy, with no
blocking, fusion or reordering beyond the definition. The bf16 inputs are widened to fp64
exactly by the caller. Sources:

  [CRISP]  "CRISP: Cliff-awaRe Input-adaptive Sparse Prefilling with Structural-Mass-Motivated
           Routing" (paper text): §2 sparse attention on an index set and the proxy attention
           over a representative query subset; §3.2 the C_struct routing signal; §4 the noise
           floor mu and the keep rule, with both directions (vertical, slash) kept; §5 setup.
  [BLOG]   rcap.io post "CRISP: Cliff-aware Input-adaptive Sparse Prefilling with ...",
           per-head pseudocode (proxy attention, C_struct, VS noise floor, PE gamma cumsum).

Readings where the pages leave a step open (each also listed in the design notes):
  R1 the proxy attention is causal: query row r (absolute position n-B+r) sees keys j <= n-B+r;
  R2 recency anchors are the fixed last `anchors` keys, the sink anchors the first `anchors`;
     C_struct is the row-mean of the mass on their union;
  R3 block pooling of the column/diagonal means is a SUM over the block, so each direction's
     block masses add up to 1 (the noise floor's 1-p[0]-p[-1] is then the residual mass);
  R4 the diagonal mean divides by B at every offset, also where fewer than B rows reach it;
  R5 keep rule uses strict '>' on blocks 1..N_b-2; anchors 0 and N_b-1 are always kept;
     min_blocks tops a direction up with its largest remaining blocks (ties: lower index);
     with N_b <= 2 every causal block is kept;
  R6 slash offset block m maps, for query block qb, to key blocks {qb-m, qb-m-1};
  R7 the PE gamma cut is one global cut over the flattened block-causal pooled matrix
     (total mass N_b), order (P desc, qb asc, kb asc), shortest prefix with cumsum >= gamma*N_b;
     every PE row also keeps {0, qb-1, qb}; gamma >= 1 keeps everything.
  R8 (FlexPrefill baseline, [CRISP] §2 and §3 discussion) the pooled estimate a_bar is the
     softmax over all N_b key blocks of mean(Q_last) . Kbar[kb] / sqrt(d); the per-query mean
     a_hat pooled to blocks is p_v; JSD uses natural logs (0 log 0 = 0); VS iff JSD >= tau;
  R9 (FlexPrefill baseline) each direction keeps the shortest prefix of its blocks sorted
     (p desc, index asc) whose sum reaches gamma times the direction's total; the first and last
     blocks are added as for CRISP (the merge of R6 is unchanged);
  R10 (median floor, [CRISP] §4 robustness discussion / Table 9) mu_d is the median of
     p_d[1..N_b-2] (mean of the two middle values when N_b-2 is even); the keep rule is unchanged.
  R11 (any length) with n not a multiple of B there are N_b = ceil(n/B) blocks and the last
     query and key blocks are partial: a block's keys are its tokens below n, block masses pool
     what the block has, block means average the rows it has; the proxy still takes the last B
     queries and the anchors are still the first and last B keys (selection needs n >= B).
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-5


# ----------------------------------------------------------------------------------------------
# Proxy attention and routing  ([CRISP] §2, §3.2; [BLOG] pseudocode)
# ----------------------------------------------------------------------------------------------
def proxy_attention(q_last: np.ndarray, k: np.ndarray, n: int) -> np.ndarray:
    """A_hat[r, j] = softmax_j(q_r . k_j / sqrt(d)) over j <= n-B+r (reading R1); zero elsewhere.

    q_last: [B, d] fp64, the queries at positions n-B .. n-1.  k: [n, d] fp64.
    """
    B, d = q_last.shape
    logits = (q_last @ k.T) / np.sqrt(d)                      # [B, n]
    pos = np.arange(n)[None, :]
    row_pos = (n - B + np.arange(B))[:, None]
    visible = pos <= row_pos
    logits = np.where(visible, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.where(visible, np.exp(logits - m), 0.0)
    return e / e.sum(axis=1, keepdims=True)


def c_struct(a_hat: np.ndarray, n: int, anchors: int) -> float:
    """Mean over proxy rows of the mass on sink [0,anchors) union recency [n-anchors, n) (R2)."""
    cols = np.zeros(n, dtype=bool)
    cols[:anchors] = True
    cols[max(n - anchors, 0):] = True
    return float(a_hat[:, cols].sum(axis=1).mean())


def route_is_vs(c: float, tau: float) -> bool:
    """Vertical-Slash iff C_struct >= tau_proxy ([CRISP] §3.2)."""
    return c >= tau


def pooled_estimate(q_last: np.ndarray, k: np.ndarray, B: int) -> np.ndarray:
    """FlexPrefill's a_bar: softmax over all key blocks of mean(q_last) . Kbar[kb] / sqrt(d) (R8)."""
    d = q_last.shape[1]
    s = (q_last.mean(axis=0) @ block_mean(k, B).T) / np.sqrt(d)
    e = np.exp(s - s.max())
    return e / e.sum()


def jsd(p: np.ndarray, q: np.ndarray) -> float:
    """Jensen-Shannon divergence (natural log): KL(p||m)/2 + KL(q||m)/2 with m = (p+q)/2."""
    m = 0.5 * (p + q)
    def kl(a):
        nz = a > 0
        return float(np.sum(a[nz] * np.log(a[nz] / m[nz])))
    return 0.5 * kl(p) + 0.5 * kl(q)


# ----------------------------------------------------------------------------------------------
# Vertical and slash scores pooled into key blocks  ([CRISP] §4, decomposition paragraph)
# ----------------------------------------------------------------------------------------------
def pool_blocks(x: np.ndarray, B: int) -> np.ndarray:
    """Sums of consecutive runs of B entries; a partial last run sums what exists (R11)."""
    nb = -(-x.shape[0] // B)
    return np.concatenate([x, np.zeros(nb * B - x.shape[0])]).reshape(nb, B).sum(axis=1)


def vertical_block_mass(a_hat: np.ndarray, B: int) -> np.ndarray:
    """p_v[b] = sum over keys of block b of the column mean of A_hat (R3)."""
    col_mean = a_hat.mean(axis=0)                             # (1/B) sum_r
    return pool_blocks(col_mean, B)


def slash_block_mass(a_hat: np.ndarray, n: int, B: int) -> np.ndarray:
    """p_s[m] = sum over offsets o in [mB, mB+B) of the diagonal mean a_s[o] (R3, R4).

    a_s[o] = (1/B) * sum over rows r with i_r - o >= 0 of A_hat[r, i_r - o],  i_r = n-B+r.
    """
    a_s = np.zeros(n)
    for r in range(B):
        i_r = n - B + r
        # offsets 0..i_r read the row backwards from the diagonal
        a_s[: i_r + 1] += a_hat[r, i_r::-1]
    a_s /= B
    return pool_blocks(a_s, B)


# ----------------------------------------------------------------------------------------------
# Noise floor and keep set  ([CRISP] §4; [BLOG] pseudocode)
# ----------------------------------------------------------------------------------------------
def noise_floor(p: np.ndarray) -> float:
    """mu = max(1 - p[0] - p[-1], 0) / (N_b - 2): mean residual mass of the non-anchor blocks."""
    nb = p.shape[0]
    return max(1.0 - p[0] - p[-1], 0.0) / (nb - 2)


def median_floor(p: np.ndarray) -> float:
    """mu = median of the non-anchor block masses p[1..N_b-2] (R10)."""
    return float(np.median(p[1:-1]))


def gamma_keep_direction(p: np.ndarray, gamma: float) -> tuple[list[int], float]:
    """FlexPrefill's per-direction rule (R9): the shortest prefix of the blocks sorted (p desc,
    j asc) whose sum reaches gamma * sum(p). Returns (kept blocks in [1, N_b-2], cut value)."""
    nb = p.shape[0]
    order = np.lexsort((np.arange(nb), -p))
    csum = np.cumsum(p[order])
    hit = np.nonzero(csum >= gamma * p.sum())[0]
    count = int(hit[0]) + 1 if hit.size else nb
    kept = order[:count]
    return sorted(int(j) for j in kept if 1 <= j <= nb - 2), float(p[order[count - 1]])


def keep_blocks(p: np.ndarray, alpha: float, min_blocks: int = 0, floor: str = "mean") -> list[int]:
    """Blocks j in [1, N_b-2] with p[j] > alpha*mu (strict), topped up to min_blocks (R5);
    mu is the mean floor of [CRISP] §4 or the median floor (R10)."""
    nb = p.shape[0]
    mu = noise_floor(p) if floor == "mean" else median_floor(p)
    keep = [j for j in range(1, nb - 1) if p[j] > alpha * mu]
    return top_up(p, keep, min_blocks)


def top_up(p: np.ndarray, keep: list[int], min_blocks: int) -> list[int]:
    """Add the largest remaining blocks of [1, N_b-2] (ties: lower index) up to min_blocks (R5)."""
    nb = p.shape[0]
    if min_blocks > len(keep):
        rest = [j for j in range(1, nb - 1) if j not in set(keep)]
        rest.sort(key=lambda j: (-p[j], j))
        keep = sorted(keep + rest[: min_blocks - len(keep)])
    return keep


def merge_vertical_slash(keep_v, keep_s, nb: int) -> list[np.ndarray]:
    """Per query block qb, the sorted key blocks of a VS head (R5, R6).

    S(qb) = ({0} u {j in keep_v u {N_b-1} : j <= qb} u U_{m in keep_s u {0, N_b-1}} {qb-m, qb-m-1})
            intersected with [0, qb].
    """
    if nb <= 2:
        return [np.arange(qb + 1) for qb in range(nb)]
    verts = set(keep_v) | {nb - 1}
    slash = set(keep_s) | {0, nb - 1}
    out = []
    for qb in range(nb):
        s = {0}
        s |= {j for j in verts if j <= qb}
        for m in slash:
            s |= {qb - m, qb - m - 1}
        out.append(np.array(sorted(j for j in s if 0 <= j <= qb), dtype=np.int64))
    return out


# ----------------------------------------------------------------------------------------------
# Pooled-Estimation path  ([CRISP] §2 and §4 PE paragraph; [BLOG] gamma_cumsum(pool(Q), pool(K)))
# ----------------------------------------------------------------------------------------------
def block_mean(x: np.ndarray, B: int) -> np.ndarray:
    """Mean of each block of B consecutive rows: [n, d] -> [ceil(n/B), d]; a partial last block
    is the mean of the rows it has (R11)."""
    n = x.shape[0]
    return np.stack([x[i:min(i + B, n)].mean(axis=0) for i in range(0, n, B)])


def pooled_scores(q: np.ndarray, k: np.ndarray, B: int) -> np.ndarray:
    """P[qb, kb] = softmax over kb <= qb of (Qbar[qb] . Kbar[kb] / sqrt(d)); zero above diagonal."""
    d = q.shape[1]
    qbar, kbar = block_mean(q, B), block_mean(k, B)
    s = (qbar @ kbar.T) / np.sqrt(d)
    nb = s.shape[0]
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    s = np.where(causal, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.where(causal, np.exp(s - m), 0.0)
    return e / e.sum(axis=1, keepdims=True)


def gamma_cut(scores: np.ndarray, gamma: float, total: float):
    """Shortest prefix of `scores` sorted (value desc, then index asc) whose cumsum >= gamma*total.

    Returns (kept indices into `scores`, sort order, cumsum-before of each sorted entry).
    gamma >= 1 keeps everything (R7).
    """
    order = np.lexsort((np.arange(scores.shape[0]), -scores))
    sorted_vals = scores[order]
    csum = np.cumsum(sorted_vals)
    before = csum - sorted_vals
    if gamma >= 1.0:
        return order, order, before
    target = gamma * total
    hit = np.nonzero(csum >= target)[0]
    count = int(hit[0]) + 1 if hit.size else scores.shape[0]
    return order[:count], order, before


def pe_select(q: np.ndarray, k: np.ndarray, B: int, gamma: float):
    """Index lists of a PE head plus the tie information of its global cut (R7)."""
    P = pooled_scores(q, k, B)
    nb = P.shape[0]
    qi, ki = np.tril_indices(nb)                              # row-major: qb asc, then kb asc
    flat = P[qi, ki]
    kept, order, before = gamma_cut(flat, gamma, float(nb))
    sel = np.zeros((nb, nb), dtype=bool)
    sel[qi[kept], ki[kept]] = True
    for qb in range(nb):
        for j in (0, qb - 1, qb):
            if 0 <= j <= qb:
                sel[qb, j] = True
    lists = [np.nonzero(sel[qb, : qb + 1])[0].astype(np.int64) for qb in range(nb)]
    # tie band: scores within TIE_REL of the cut entry, or cumsum-before within TIE_REL of target
    ties = np.zeros((nb, nb), dtype=bool)
    if gamma < 1.0 and kept.shape[0] < flat.shape[0]:
        cut_val = flat[kept[-1]]
        target = gamma * nb
        near_val = np.abs(flat - cut_val) <= TIE_REL * cut_val
        near_sum = np.zeros_like(near_val)
        near_sum[order] = np.abs(before - target) <= TIE_REL * target
        t = near_val | near_sum
        ties[qi[t], ki[t]] = True
    return lists, P, ties


# ----------------------------------------------------------------------------------------------
# Per-head selection  ([BLOG] per-head flow; [CRISP] §3.2, §4)
# ----------------------------------------------------------------------------------------------
JSD_TIE_REL = TIE_REL  # the routing band is the same 1e-5 relative band as every other threshold


def select_head(q: np.ndarray, k: np.ndarray, *, block=128, anchors=128, tau_proxy=0.5,
                alpha=1.0, gamma=0.95, min_blocks=0, route_rule="cstruct", tau_jsd=0.1,
                vs_rule="floor", floor="mean") -> dict:
    """Route one q-head and build its per-query-block key-block lists.

    q: [n, d] fp64 queries of the head; k: [n, d] fp64 keys of its kv-head.
    CRISP: route_rule="cstruct", vs_rule="floor" (floor="mean", or "median" for R10).
    FlexPrefill baseline: route_rule="jsd" (R8), vs_rule="gamma" (R9).
    """
    n = q.shape[0]
    B = block
    nb = -(-n // B)                     # partial last block when n is not a multiple of B (R11)
    a_hat = proxy_attention(q[n - B:], k, n)
    c = c_struct(a_hat, n, anchors)
    p_v = vertical_block_mass(a_hat, B)
    p_s = slash_block_mass(a_hat, n, B)
    out = dict(c_struct=c, p_v=p_v, p_s=p_s)
    if route_rule == "jsd":
        j = jsd(pooled_estimate(q[n - B:], k, B), p_v)
        vs = j >= tau_jsd
        out.update(jsd=j, route_tie=abs(j - tau_jsd) <= JSD_TIE_REL * tau_jsd)
    else:
        vs = route_is_vs(c, tau_proxy)
        out["route_tie"] = abs(c - tau_proxy) <= TIE_REL * tau_proxy
    out["route"] = int(vs)
    if nb >= 3:
        if floor == "median":
            out["mu_v"], out["mu_s"] = median_floor(p_v), median_floor(p_s)
        else:
            out["mu_v"], out["mu_s"] = noise_floor(p_v), noise_floor(p_s)
    if vs:
        if nb <= 2:
            out["lists"] = [np.arange(qb + 1) for qb in range(nb)]
            out["keep_v"], out["keep_s"] = [], []
            out["vs_ties_v"], out["vs_ties_s"] = [], []
        elif vs_rule == "gamma":
            for name, p in (("v", p_v), ("s", p_s)):
                kept, cut = gamma_keep_direction(p, gamma)
                out["keep_" + name] = top_up(p, kept, min_blocks)
                # ties: values within TIE_REL of the cut value, or a prefix sum within TIE_REL of
                # the target (either can flip with rounding)
                order = np.lexsort((np.arange(nb), -p))
                before = np.cumsum(p[order]) - p[order]
                target = gamma * p.sum()
                near = set(int(order[i]) for i in range(nb) if abs(before[i] - target) <= TIE_REL * target)
                near |= {jj for jj in range(nb) if abs(p[jj] - cut) <= TIE_REL * cut}
                out["vs_ties_" + name] = sorted(jj for jj in near if 1 <= jj <= nb - 2)
            out["lists"] = merge_vertical_slash(out["keep_v"], out["keep_s"], nb)
        else:
            keep_v = keep_blocks(p_v, alpha, min_blocks, floor)
            keep_s = keep_blocks(p_s, alpha, min_blocks, floor)
            out["keep_v"], out["keep_s"] = keep_v, keep_s
            out["lists"] = merge_vertical_slash(keep_v, keep_s, nb)
            for name, p, mu in (("v", p_v, out["mu_v"]), ("s", p_s, out["mu_s"])):
                thr = alpha * mu
                band = max(TIE_REL * thr, 1e-30)
                out["vs_ties_" + name] = [j for j in range(1, nb - 1) if abs(p[j] - thr) <= band]
    else:
        lists, P, ties = pe_select(q, k, B, gamma)
        out["lists"], out["pe_scores"], out["pe_ties"] = lists, P, ties
    return out


# ----------------------------------------------------------------------------------------------
# Attention on an index set  ([CRISP] §2: softmax(QK^T/sqrt(d) + M_S) V)
# ----------------------------------------------------------------------------------------------
def attention_block(q_blk: np.ndarray, k: np.ndarray, v: np.ndarray, key_blocks, qb: int, B: int = 128):
    """Output rows of query block qb (queries q_blk = q[qb*B:(qb+1)*B]) attending to the keys of
    `key_blocks`, causally: O[i] = sum_{j in S(qb), j <= i} softmax_j(q_i . k_j / sqrt(d)) v_j.
    Returns (O [B, d], lse [B]) with lse the natural-log sum of exp of the scaled logits.
    """
    d = q_blk.shape[1]
    n = k.shape[0]
    # the last block of a sequence whose length is not a multiple of B is partial (R11)
    keys = np.concatenate([np.arange(kb * B, min(kb * B + B, n)) for kb in key_blocks])
    rows = np.arange(qb * B, qb * B + q_blk.shape[0])
    s = (q_blk @ k[keys].T) / np.sqrt(d)
    allowed = keys[None, :] <= rows[:, None]
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.where(allowed, np.exp(s - m), 0.0)
    z = e.sum(axis=1, keepdims=True)
    return (e / z) @ v[keys], (m + np.log(z))[:, 0]


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_blocks, qb: int, B: int = 128):
    """attention_block for query block qb of a full query matrix q [n, d]."""
    return attention_block(q[qb * B:(qb + 1) * B], k, v, key_blocks, qb, B)


def attention_head(q, k, v, lists, B: int = 128):
    """Full output of one head for per-query-block key-block lists."""
    n = q.shape[0]
    o = np.zeros_like(q)
    lse = np.zeros(n)
    for qb, kb in enumerate(lists):
        o[qb * B:(qb + 1) * B], lse[qb * B:(qb + 1) * B] = attention_rows(q, k, v, kb, qb, B)
    return o, lse


def dense_causal_attention(q, k, v):
    """Exact causal softmax attention over all keys j <= i (no blocking)."""
    n, d = q.shape
    s = (q @ k.T) / np.sqrt(d)
    s = np.where(np.tril(np.ones((n, n), dtype=bool)), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return (e / e.sum(axis=1, keepdims=True)) @ v


# ----------------------------------------------------------------------------------------------
# FP8 variant of the attention logits: Q and K quantised to 8-bit E4M3 per 128-row block
# (the OCP 8-bit floating-point format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
# no infinities, largest finite value 448, subnormals m * 2^-9). The attention itself is then the
# exact attention of the dequantised Q and K (attention_rows on them).
# ----------------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """Value of each E4M3 code (uint8); the two NaN codes (0x7f, 0xff) decode to nan."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 0xF) & (m == 0x7), np.nan, mag)
    return sign * mag


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """Round each value to the nearest E4M3 value, ties to the even code, saturating at +-448
    (finite inputs); the sign bit is the input's, so small negative values give -0 (0x80). Written from the format: the representable magnitudes are enumerated and the
    nearest one is picked, so no rounding arithmetic can be wrong here."""
    y = np.asarray(y, dtype=np.float64)
    codes = np.arange(0x7F, dtype=np.int64)                  # 0x00 .. 0x7e: every finite magnitude
    mags = e4m3_decode(codes)                                # ascending
    a = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.searchsorted(mags, a, side="left").clip(0, len(mags) - 1)
    lo = (hi - 1).clip(0, None)
    d_hi = np.abs(mags[hi] - a)
    d_lo = np.abs(a - mags[lo])
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = d_lo == d_hi
    pick = np.where(tie & (lo != hi), np.where(codes[lo] % 2 == 0, lo, hi), pick)
    out = codes[pick]
    out = np.where(np.signbit(y), out | 0x80, out)          # the sign is kept, also on zero
    return out.astype(np.uint8)


def quantize_blocks_fp8(x: np.ndarray, B: int = 128):
    """Per block of B rows of x [n, d] (bf16 values widened exactly): amax = max |x| in fp32,
    codes = E4M3(fp32(x) * fp32(448 / amax)) with the product and quotient rounded to fp32, and the
    dequantisation scale fp32(amax / 448); an all-zero block gets codes 0 and scale 1. Returns
    (codes uint8 [n, d], scales float32 [N_b]); the dequantised block is e4m3_decode(codes) * scale."""
    n = x.shape[0]
    nb = -(-n // B)
    xs = np.asarray(x, dtype=np.float32)
    codes = np.zeros(xs.shape, dtype=np.uint8)
    scales = np.ones(nb, dtype=np.float32)
    for b in range(nb):
        blk = xs[b * B:min(n, (b + 1) * B)]
        amax = np.float32(np.abs(blk).max()) if blk.size else np.float32(0)
        if amax == 0:
            continue
        inv = np.float32(np.float32(E4M3_MAX) / amax)
        codes[b * B:min(n, (b + 1) * B)] = e4m3_encode((blk * inv).astype(np.float32))
        scales[b] = np.float32(amax / np.float32(E4M3_MAX))
    return codes, scales


def dequantize_blocks_fp8(codes: np.ndarray, scales: np.ndarray, B: int = 128) -> np.ndarray:
    """fp64 values of the quantised blocks: e4m3_decode(code) * scale of the row's block."""
    vals = e4m3_decode(codes)
    rows = np.arange(codes.shape[0]) // B
    return vals * np.asarray(scales, dtype=np.float64)[rows][:, None]
