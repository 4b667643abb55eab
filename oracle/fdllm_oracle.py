"""Plain fp64 CPU oracle for the Flash-dLLM fused KV-cache step.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke entry and the
benchmark's CPU-baseline / reference leg may import this module.  The product
path (the CUDA library and its binding) never calls it and shares no code with
it; the two meet only through the seeded inputs of the `workloads` package.

Citations name the page by its title and then the section, algorithm or figure
on it:
  [review]  "Flash-dLLM: IO-Aware KV Caching and Parallel Decoding for Fast,
            Memory-Efficient Diffusion LLMs" (jaehun.me review of
            arXiv 2609.26796).
  [summary] "Flash-dLLM: IO-Aware KV Caching and Parallel Decoding for Fast
            Diffusion LLMs" (alanhou.org summary), "Core Mechanism".

What is computed (each function states its passage):
  * fused_step   - one call of the IO-aware fused KV-cache step ([review],
                   "How It Works", Step 1: Draft, Alg. 1): read only x[Q],
                   project to q,k,v, rotate q,k at their positions, write k,v
                   into the cache at Q, then attend Q over the whole cache.
  * verify_step  - the Flash-Verify pass ([review], "Flash-Verify", sec. 2.3,
                   Fig. 2; "How It Works", Step 1: Verification): rows
                   [T_v | draft view | mask view]; the two views share
                   positions, and neither view attends to the other's keys.
  * accept       - top-1 / confidence, the epsilon split into D_t / S_t and the
                   gamma prefix acceptance ([review], "Flash-Verify", sec. 2.3
                   and the worked example).
  * attention_mass, track_select - the tracked set of the next step ([review],
                   "How It Works", Step 1: Cache selection): the decoded slots
                   that receive the largest share of the masked queries'
                   attention.

Everything is computed in float64 from the exactly upcast stored inputs.  The
k,v written into the cache are rounded once to the storage dtype, and the
attention reads the cache as stored.  No blocking, fusion or reordering is used
beyond the definitions: a reader can check each line against the passage.

Readings where the pages are silent (they are listed with reasons in the
design notes): rotate-half RoPE with theta_j = base^(-2j/dh) at the absolute
cache slot; softmax scale 1/sqrt(dh); W_qkv rows are [q | k | v], head-major;
no mask in the draft pass; attention sees the newly written k,v; argmax ties
go to the lowest token index; thresholds are inclusive (c >= eps, c~ >= gamma).
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# storage formats


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns: the top 16 bits of a float32."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    bfloat16 keeps 8 significant bits.  With x = m * 2^e, 0.5 <= |m| < 1
    (frexp, exact), one unit in the last place is 2^(e-8), floored at the
    smallest subnormal step 2^-133; x / ulp is exact, so rint (ties to even)
    gives the single correctly rounded result."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp = np.ldexp(1.0, np.maximum(e - 8, -133))
    return np.rint(x / ulp) * ulp


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns of float64 values (rounded to nearest even first)."""
    r = round_bf16(x).astype(np.float32)  # exact: bf16 values are float32 values
    return (r.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype ("bf16", "f32" or "f64"), as float64."""
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(x, np.float64)
    raise ValueError(dtype)


def to_f64(t) -> np.ndarray:
    """float64 copy of a stored tensor (numpy array or torch CPU tensor of f32/f64/bf16)."""
    if hasattr(t, "dtype") and str(t.dtype) == "torch.bfloat16":
        return bf16_bits_to_f64(t.contiguous().view(dtype=_torch_int16()).numpy().view(np.uint16))
    if hasattr(t, "numpy"):
        t = t.numpy()
    return np.asarray(t, dtype=np.float64)


def _torch_int16():
    import torch  # storage decoding only
    return torch.int16


# ----------------------------------------------------------------------------
# building blocks


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotary position embedding of x [n, H, dh] at absolute positions pos [n].

    The pages only say that the two verify views share position embeddings
    ([review], "Flash-Verify", sec. 2.3).  Reading: rotate-half pairs
    (j, j + dh/2) turned by the angle pos * base^(-2j/dh), j < dh/2."""
    n, H, dh = x.shape
    half = dh // 2
    j = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * j / dh)
    ang = np.asarray(pos, np.float64)[:, None] * theta[None, :]  # [n, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def project_qkv(x_rows: np.ndarray, w_qkv: np.ndarray, H: int, dh: int):
    """q, k, v [n, H, dh] = x_rows [n, D] times W_qkv^T, W_qkv [3*H*dh, D].

    The fused kernel builds q, k, v from x[Q] on chip ([review], "How It
    Works", Step 1: Draft, Alg. 1).  Layout reading: W rows are the q block,
    then the k block, then the v block, each head-major."""
    E = H * dh
    y = x_rows @ w_qkv.T
    n = x_rows.shape[0]
    return (y[:, :E].reshape(n, H, dh), y[:, E:2 * E].reshape(n, H, dh),
            y[:, 2 * E:].reshape(n, H, dh))


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, visible: np.ndarray | None = None):
    """softmax(q K^T / sqrt(dh)) V for one head: q [nq, dh], K, V [Nk, dh].

    visible [nq, Nk] (optional) removes keys a row may not see.  Otherwise
    every query sees every key ([review], "How It Works": the draft pass
    attends over the whole cache)."""
    dh = q.shape[-1]
    s = (q @ K.T) / np.sqrt(dh)
    if visible is not None:
        s = np.where(visible, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


# ----------------------------------------------------------------------------
# the step


def fused_step(x, q_idx, w_qkv, rope_base, k_cache, v_cache, H, dh, dtype):
    """One fused KV-cache step ([review], "How It Works", Step 1: Draft, Alg. 1).

    x [B, N, D], q_idx [B, nq] (distinct slots of each sequence), w_qkv
    [3E, D], k_cache / v_cache [B, H, N, dh], all float64 values of the stored
    inputs.  For each sequence: read only the rows x[b, Q], project and rotate
    them, write k, v (rounded to `dtype`) into the cache at Q, then attend every
    query over all N slots of the updated cache.

    Returns (K', V', out) with out [B, nq, H*dh] in float64."""
    B, nq = q_idx.shape
    K2 = np.array(k_cache, dtype=np.float64, copy=True)
    V2 = np.array(v_cache, dtype=np.float64, copy=True)
    out = np.zeros((B, nq, H * dh))
    for b in range(B):
        Q = np.asarray(q_idx[b], dtype=np.int64)
        q, k, v = project_qkv(x[b, Q], w_qkv, H, dh)
        q = rope(q, Q, rope_base)
        k = rope(k, Q, rope_base)
        K2[b][:, Q, :] = round_to(k, dtype).transpose(1, 0, 2)
        V2[b][:, Q, :] = round_to(v, dtype).transpose(1, 0, 2)
        for h in range(H):
            out[b, :, h * dh:(h + 1) * dh] = attend(q[:, h], K2[b, h], V2[b, h])
    return K2, V2, out


def verify_visibility(view, rank, n_cache_pos, draft_pos, causal_cross=False):
    """Which keys each verify row may see.

    Keys are the N cache slots followed by the side slots that hold the
    mask-view k,v (one per mask-view row, in row order).  The draft view and
    the mask view share positions while each is hidden from the other ([review],
    "Flash-Verify", sec. 2.3, Fig. 2; "How It Works", Step 1: Verification):
      * view 0 (T_v) and view 1 (draft) rows see every cache slot, including
        the draft-view k,v written at the S positions, and no side slot;
      * view 2 (mask) rows see every cache slot except the S positions, and
        every side slot.
    causal_cross=True is the reading of the pages' causal remark ([review],
    Appx. C, Remark 1): a mask row of rank r sees the draft key at an S
    position of rank < r and the mask key at an S position of rank >= r.

    Returns bool [R, N + n_side]."""
    view = np.asarray(view)
    rank = np.asarray(rank)
    R = view.shape[0]
    mask_rows = np.nonzero(view == 2)[0]
    n_side = len(mask_rows)
    side_rank = rank[mask_rows]
    dpos = np.asarray(draft_pos[0], np.int64)
    drank = np.asarray(draft_pos[1])
    vis = np.zeros((R, n_cache_pos + n_side), dtype=bool)
    for r in range(R):
        if view[r] in (0, 1):
            vis[r, :n_cache_pos] = True
        elif view[r] == 2:
            vis[r, :n_cache_pos] = True
            if causal_cross:
                vis[r, dpos] = drank < rank[r]
                vis[r, n_cache_pos:] = side_rank >= rank[r]
            else:
                vis[r, dpos] = False
                vis[r, n_cache_pos:] = True
        else:
            raise ValueError("view must be 0, 1 or 2")
    return vis


def verify_step(x_rows, pos, view, rank, w_qkv, rope_base, k_cache, v_cache,
                k_side, v_side, H, dh, dtype, causal_cross=False):
    """One Flash-Verify pass over packed rows ([review], "Flash-Verify", sec. 2.3).

    x_rows [B, R, D]; pos, view, rank [B, R]; caches [B, H, N, dh]; side
    buffers [B, H, S_max, dh].  Rows of view 0 (T_v) and view 1 (draft) write
    their k,v into the cache at pos; rows of view 2 (mask) write theirs into
    side slots 0, 1, ... in row order, so the cache never holds [MASK]-view
    keys.  Every row then attends over the keys verify_visibility allows.

    Returns (K', V', K_side', V_side', out [B, R, H*dh])."""
    B, R = pos.shape
    N = k_cache.shape[2]
    K2 = np.array(k_cache, dtype=np.float64, copy=True)
    V2 = np.array(v_cache, dtype=np.float64, copy=True)
    KS = np.array(k_side, dtype=np.float64, copy=True)
    VS = np.array(v_side, dtype=np.float64, copy=True)
    out = np.zeros((B, R, H * dh))
    for b in range(B):
        P = np.asarray(pos[b], np.int64)
        vw = np.asarray(view[b])
        q, k, v = project_qkv(x_rows[b], w_qkv, H, dh)
        q = rope(q, P, rope_base)
        k = rope(k, P, rope_base)
        kr = round_to(k, dtype)
        vr = round_to(v, dtype)
        in_cache = np.nonzero((vw == 0) | (vw == 1))[0]
        K2[b][:, P[in_cache], :] = kr[in_cache].transpose(1, 0, 2)
        V2[b][:, P[in_cache], :] = vr[in_cache].transpose(1, 0, 2)
        mask_rows = np.nonzero(vw == 2)[0]
        for s, r in enumerate(mask_rows):
            KS[b][:, s, :] = kr[r]
            VS[b][:, s, :] = vr[r]
        drows = np.nonzero(vw == 1)[0]
        vis = verify_visibility(vw, rank[b], N, (P[drows], np.asarray(rank[b])[drows]),
                                causal_cross)
        n_side = len(mask_rows)
        for h in range(H):
            Kall = np.concatenate([K2[b, h], KS[b, h, :n_side]], axis=0)
            Vall = np.concatenate([V2[b, h], VS[b, h, :n_side]], axis=0)
            out[b, :, h * dh:(h + 1) * dh] = attend(q[:, h], Kall, Vall, vis)
    return K2, V2, KS, VS, out


# ----------------------------------------------------------------------------
# acceptance

FLAG_COMMIT = 1    # kind 1 row with confidence >= eps: joins D_t
FLAG_ACCEPT = 2    # kind 2 row accepted by the gamma prefix rule
FLAG_PASS = 4      # kind 2 row whose own test passed (top-1 agrees, conf >= gamma)


def accept(logits, kind, ref_tok, rank, eps, gamma):
    """Top-1, confidence, epsilon split and gamma prefix acceptance.

    logits [B, R, V] (float64 values of the fp32 logits); kind, ref_tok, rank
    [B, R].  Per row ([review], "Flash-Verify", sec. 2.3):
      * top1 = the lowest token index attaining the largest logit, and the
        confidence c = max_v softmax(logits)_v = 1 / sum_v exp(l_v - l_max);
      * kind 1 (draft-pass masked row): FLAG_COMMIT iff c >= eps (D_t; the
        rest form S_t);
      * kind 2 (mask-view row): FLAG_PASS iff top1 == ref_tok (the draft
        prediction) and c >= gamma; the rows are taken in decoding order
        (ascending rank) and accepted up to the first one that fails
        (FLAG_ACCEPT iff rank < the smallest rank of a failing kind-2 row).
      * kind 0: top1 and c only.
    Returns (top1 [B,R] int64, conf [B,R] float64, flags [B,R] uint8, n_accept [B])."""
    logits = np.asarray(logits, np.float64)
    B, R, _ = logits.shape
    top1 = np.zeros((B, R), np.int64)
    conf = np.zeros((B, R))
    flags = np.zeros((B, R), np.uint8)
    n_accept = np.zeros(B, np.int64)
    for b in range(B):
        first_fail = np.inf
        for r in range(R):
            l = logits[b, r]
            m = l.max()
            top1[b, r] = int(np.argmax(l))  # first index attaining the max
            conf[b, r] = 1.0 / np.exp(l - m).sum()
            if kind[b, r] == 1 and conf[b, r] >= eps:
                flags[b, r] |= FLAG_COMMIT
            if kind[b, r] == 2:
                if top1[b, r] == ref_tok[b, r] and conf[b, r] >= gamma:
                    flags[b, r] |= FLAG_PASS
                else:
                    first_fail = min(first_fail, rank[b, r])
        for r in range(R):
            if kind[b, r] == 2 and rank[b, r] < first_fail:
                flags[b, r] |= FLAG_ACCEPT
                n_accept[b] += 1
    return top1, conf, flags, n_accept


# ----------------------------------------------------------------------------
# tracked-set selection


def attention_mass(x, q_idx, w_qkv, rope_base, k_cache2, H, dh, masked_row):
    """Attention mass of every cache slot ([review], "How It Works", Step 1:
    Cache selection, which ranks decoded tokens by how much the masked queries
    attend to them).

    Reading: a[b, j] = sum over the masked-query rows i of Q (masked_row[b, i]
    != 0) and over the heads h of softmax_j(q_ih . K'_hj / sqrt(dh)), the
    softmax taken over all N slots of the cache K' the step left (k_cache2,
    after the write at Q), exactly the probabilities of the draft pass.  q is
    the step's query: x[b, Q] projected and rotated at Q.  Returns [B, N]."""
    B, nq = q_idx.shape
    N = k_cache2.shape[2]
    a = np.zeros((B, N))
    for b in range(B):
        Q = np.asarray(q_idx[b], dtype=np.int64)
        rows = np.nonzero(np.asarray(masked_row[b]) != 0)[0]
        if rows.size == 0:
            continue
        q, _, _ = project_qkv(x[b, Q[rows]], w_qkv, H, dh)
        q = rope(q, Q[rows], rope_base)
        for h in range(H):
            s = (q[:, h] @ k_cache2[b, h].T) / np.sqrt(dh)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            a[b] += p.sum(axis=0)
    return a


def track_select(a, candidate, beta_t):
    """The next tracked set T ([review], "How It Works", Step 1: Cache
    selection): the beta_t candidate slots with the largest attention mass.

    candidate[b, j] != 0 marks a decoded slot.  The positions decoded in this
    step are candidates like the earlier ones (on the page, the positions
    resolved in the step take part in the ranking and T keeps beta_t
    entries).  Order: mass
    descending, equal mass to the lower slot.  With fewer candidates than
    beta_t the tail is -1.  Returns int64 [B, beta_t]."""
    B, N = a.shape
    out = np.full((B, beta_t), -1, dtype=np.int64)
    for b in range(B):
        cand = [j for j in range(N) if candidate[b, j] != 0]
        cand.sort(key=lambda j: (-a[b, j], j))
        for t, j in enumerate(cand[:beta_t]):
            out[b, t] = j
    return out
