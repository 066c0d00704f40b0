"""Plain, slow, float64 CPU oracle of the SPECTRA latent KV-cache codec.

TEST INFRASTRUCTURE: imported only by ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline legs.  It shares no code with the CUDA library.

Sources (cited by page title and section):

* [SPECTRA] "SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff via Spectral
  Transform Coding", technical summary: "Methodology" (observations 1-3),
  "SPECTRA pipeline" stage 1 (G-weighted transform, W_O refinement), stage 2
  (rate-distortion quantisation by reverse water-filling, grouping), stage 3
  (system integration: project down, quantise per token, append, rebuild K/V for
  standard attention), "Significance and claims" (attention in latent space).
* [SKV] "Spectral-KV: SVD-projection KV cache compression (28x)", "Technical
  principle" 1 (spectral profiling, K = U S V^T, energy ratio) and 2
  (k_latent = k . V_r).
* Textbook reverse water-filling for independent Gaussian sources (Cover &
  Thomas, Elements of Information Theory, ch. 10): D_i = min(theta, s_i^2),
  R_i = max(0, 1/2 log2(s_i^2/theta)).

Readings of points the pages leave open:

* G is the mean E[h^T h]; the Gram's scale leaves the basis unchanged.
* A latent coordinate's "variance" is its second moment s_i^2 (G is uncentred).
* Grouped widths: the exact minimiser of the water-filling distortion model
  sum_j S_j 4^-b_j (S_j = variance mass of group j; b = 0 drops the group) under
  the bit budget, b_j in {0,1,2,3,4,8}, by dynamic programming over groups; ties
  go to the smaller width.
* Per token and group: fp16 min-max scale s = fp16((max-min)/(2^b-1)) and fp16
  zero z = fp16(min), both saturated to +-65504; code = clamp(rne((x-z)/s)) with
  every step in IEEE fp32; s == 0 gives all-zero codes; dequantised value
  code*s + z.
* Attention: scores q.k/sqrt(d_h) against the rebuilt keys, exact softmax over
  every cached token, GQA map q head h -> KV head h // (H_q/H_kv).
* W_O correction: per q head least squares mapping the rank-truncated attention
  output onto the exact one on calibration data (the pages give no formula).
* Alternatives for the allocation ablation: uniform widths (the leading k groups
  at one width, (k, b) minimising the same model) and an energy-threshold rank
  limiting which groups may get bits.

Pinned by the ``-m "not gpu"`` tests in tests/test_oracle_*.py, except where a
function's docstring says "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

WIDTHS = (0, 1, 2, 3, 4, 8)
SIDES = ("K", "V")
FP16_MAX = 65504.0


# ----------------------------------------------------------------------------
# Calibration: Gram, whitened SVD, energy-ordered basis      [SPECTRA] stage 1
# ----------------------------------------------------------------------------

def gram(H: np.ndarray) -> np.ndarray:
    """G = E[h^T h] over the calibration tokens ([SPECTRA] observation 3), fp64."""
    H64 = np.asarray(H, dtype=np.float64)
    return (H64.T @ H64) / H64.shape[0]


def psd_sqrt(G: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(G^{1/2}, G^{-1/2}) of a symmetric positive definite G via eigh."""
    lam, Q = np.linalg.eigh((G + G.T) / 2)
    if lam.min() <= 0:
        raise ValueError("Gram matrix is not positive definite")
    return (Q * np.sqrt(lam)) @ Q.T, (Q / np.sqrt(lam)) @ Q.T


def sign_fix(V: np.ndarray) -> np.ndarray:
    """Flip each column so its largest-magnitude entry (lowest index on ties) is > 0."""
    V = np.array(V, dtype=np.float64, copy=True)
    idx = np.argmax(np.abs(V), axis=0)
    sgn = np.sign(V[idx, np.arange(V.shape[1])])
    sgn[sgn == 0] = 1.0
    return V * sgn[None, :]


def whitened_svd(G: np.ndarray, W: np.ndarray, r: int) -> dict:
    """The G-weighted SVD of [SPECTRA] stage 1, written out literally.

    SVD of G^{1/2} W = U S V^T (the weights whitened by the activation Gram), sorted
    by decreasing singular value.  Returns V (d_h x d_h), sigma2 = S^2 (the
    latent second moments), W_down = G^{-1/2} U_r S_r and W_up = V_r^T.  W_down
    equals W V_r; the function checks that.
    """
    W = np.asarray(W, dtype=np.float64)
    Gh, Gih = psd_sqrt(G)
    U, S, Vt = np.linalg.svd(Gh @ W, full_matrices=False)
    order = np.argsort(-S, kind="stable")
    U, S, V = U[:, order], S[order], Vt.T[:, order]
    Vf = sign_fix(V)
    flip = np.sign(np.sum(Vf * V, axis=0))
    U = U * flip[None, :]
    V = Vf
    W_down = (Gih @ U[:, :r]) * S[None, :r]
    W_down_fold = W @ V[:, :r]
    err = np.abs(W_down - W_down_fold).max() / max(np.abs(W_down_fold).max(), 1e-300)
    if err > 1e-8:
        raise AssertionError(f"G^-1/2 U S != W V_r (rel {err:.3e})")
    return dict(V=V, sigma2=S ** 2, W_down=W_down_fold, W_up=V[:, :r].T, U=U, S=S)


def latent_basis(G: np.ndarray, W: np.ndarray, r: int) -> dict:
    """Same basis from the closed form: G^{1/2}W = U S V^T  =>  W^T G W = V S^2 V^T.

    eigh of the d_h x d_h matrix M = W^T G W, eigenvalues sorted decreasing,
    eigenvector signs fixed by ``sign_fix``.
    """
    W = np.asarray(W, dtype=np.float64)
    M = W.T @ G @ W
    M = (M + M.T) / 2
    lam, V = np.linalg.eigh(M)
    order = np.argsort(-lam, kind="stable")
    lam, V = lam[order], sign_fix(V[:, order])
    return dict(V=V, sigma2=np.clip(lam, 0.0, None), W_down=W @ V[:, :r], W_up=V[:, :r].T)


def keys_svd_basis(H: np.ndarray, W: np.ndarray, r: int) -> dict:
    """[SKV] route: SVD of the calibration keys K = H W = U S V^T, k_latent = k V_r.

    With G = H^T H / N this gives the same V, and S_i^2 = N sigma_i^2.
    """
    K = np.asarray(H, dtype=np.float64) @ np.asarray(W, dtype=np.float64)
    _, S, Vt = np.linalg.svd(K, full_matrices=False)
    order = np.argsort(-S, kind="stable")
    V = sign_fix(Vt.T[:, order])
    return dict(V=V, sigma2=S[order] ** 2 / K.shape[0], W_up=V[:, :r].T)


# ----------------------------------------------------------------------------
# Bit allocation: reverse water-filling and grouped widths    [SPECTRA] stage 2
# ----------------------------------------------------------------------------

def reverse_water_fill(sigma2: np.ndarray, R: float, tol: float = 1e-14) -> dict:
    """Continuous reverse water-filling: find theta with sum_i R_i = R.

    R_i = max(0, 1/2 log2(sigma_i^2/theta)), D_i = min(theta, sigma_i^2).  Bisection
    on log(theta) to ``tol`` relative.  R = 0 gives theta = max sigma^2.
    """
    s2 = np.asarray(sigma2, dtype=np.float64)
    pos = s2[s2 > 0]
    if R <= 0 or pos.size == 0:
        theta = float(s2.max()) if s2.size else 0.0
        return dict(theta=theta, R=np.zeros_like(s2), D=np.minimum(theta, s2))

    def rate(log_t):
        return np.maximum(0.0, 0.5 * (np.log2(pos) - log_t / math.log(2))).sum()

    hi = math.log(pos.max())
    lo = math.log(pos.min()) - 2.0 * R * math.log(2) / 1.0 - 1.0
    while rate(lo) < R:
        lo -= 10.0
    for _ in range(400):
        mid = 0.5 * (lo + hi)
        if rate(mid) > R:
            lo = mid
        else:
            hi = mid
        if hi - lo < tol:
            break
    theta = math.exp(0.5 * (lo + hi))
    Ri = np.where(s2 > 0, np.maximum(0.0, 0.5 * np.log2(np.where(s2 > 0, s2, 1.0) / theta)), 0.0)
    return dict(theta=theta, R=Ri, D=np.minimum(theta, s2))


def group_cost(b: int, g: int, count_overhead: bool) -> int:
    """Bits one token spends on a group of g coordinates at width b."""
    if b == 0:
        return 0
    return g * b + (32 if count_overhead else 0)


def group_mass(sigma2: np.ndarray, g: int) -> np.ndarray:
    """S_j = sum of sigma_i^2 over group j, summed in ascending coordinate order."""
    s2 = np.asarray(sigma2, dtype=np.float64)
    n = s2.size // g
    out = np.zeros(n)
    for j in range(n):
        acc = 0.0
        for i in range(j * g, (j + 1) * g):
            acc += float(s2[i])
        out[j] = acc
    return out


def group_distortion(S_j: float, b: int) -> float:
    """Model distortion of a group at width b: S_j 2^{-2b}; b = 0 drops it (S_j)."""
    return S_j * (4.0 ** (-b))


def allocate_widths(sigma2: np.ndarray, g: int, budget: int, count_overhead: bool) -> np.ndarray:
    """Grouped widths b_j in {0,1,2,3,4,8} minimising sum_j S_j 4^-b_j.

    Constraint sum_j cost(b_j) <= budget.  Backward dynamic programme over groups
    j = n-1..0 and remaining budget c: V[j][c] = min_b S_j 4^-b + V[j+1][c-cost(b)],
    candidates tried in increasing b with strict improvement (ties -> smaller b),
    sums formed right-nested in fp64.
    """
    S = group_mass(sigma2, g)
    n = S.size
    INF = float("inf")
    V = [[0.0] * (budget + 1) for _ in range(n + 1)]
    choice = [[0] * (budget + 1) for _ in range(n)]
    for j in range(n - 1, -1, -1):
        for c in range(budget + 1):
            best, best_b = INF, 0
            for b in WIDTHS:
                cost = group_cost(b, g, count_overhead)
                if cost > c:
                    continue
                v = group_distortion(S[j], b) + V[j + 1][c - cost]
                if v < best:
                    best, best_b = v, b
            V[j][c] = best
            choice[j][c] = best_b
    widths = np.zeros(n, dtype=np.int64)
    c = budget
    for j in range(n):
        b = choice[j][c]
        widths[j] = b
        c -= group_cost(b, g, count_overhead)
    return widths


def allocate_widths_uniform(sigma2: np.ndarray, g: int, budget: int, count_overhead: bool,
                            n_eligible: int | None = None) -> np.ndarray:
    """One width for every kept group ([ABL] "Practical recommendations":
    SpectralQuant with uniform allocation).

    Reading: the kept groups are the leading k of the first n_eligible groups,
    all at one width b in {1,2,3,4,8}; among all (k, b) with k * cost(b) <= budget
    choose the least model distortion sum_j S_j 4^-b_j (k = 0 keeps nothing); ties
    go to fewer bits, then to fewer groups.  Enumerates every (k, b).
    """
    S = group_mass(sigma2, g)
    n = S.size
    ne = n if n_eligible is None else max(0, min(int(n_eligible), n))
    best = (float(sum(S)), 0, 0, 0)  # (distortion, bits, k, b)
    for b in WIDTHS[1:]:
        cost = group_cost(b, g, count_overhead)
        for k in range(1, ne + 1):
            if k * cost > budget:
                break
            w = [b] * k + [0] * (n - k)
            cand = (allocation_distortion(sigma2, w, g), k * cost, k, b)
            if cand[:3] < best[:3]:
                best = cand
    _, _, k, b = best
    return np.array([b] * k + [0] * (n - k), dtype=np.int64)


def energy_rank(sigma2: np.ndarray, threshold: float) -> int:
    """Smallest r with sum_{i<r} sigma2_i >= threshold * sum_i sigma2_i ([SKV]
    "Technical principle" 1: the effective rank at a target energy, e.g. 0.95);
    sigma2 in decreasing order, threshold in (0, 1]."""
    s2 = np.asarray(sigma2, dtype=np.float64)
    if not 0.0 < threshold <= 1.0:
        raise ValueError("threshold must be in (0, 1]")
    total = float(s2.sum())
    acc = 0.0
    for i, v in enumerate(s2):
        acc += float(v)
        if acc >= threshold * total:
            return i + 1
    return s2.size


def allocation_distortion(sigma2, widths, g) -> float:
    S = group_mass(sigma2, g)
    return float(sum(group_distortion(S[j], int(b)) for j, b in enumerate(widths)))


# ----------------------------------------------------------------------------
# Codec: factors folded per head and side                      [SPECTRA] stage 3
# ----------------------------------------------------------------------------

def nonzero_coords(widths: np.ndarray, g: int) -> np.ndarray:
    """Latent coordinate indices kept (groups with b > 0), ascending."""
    return np.concatenate([np.arange(j * g, (j + 1) * g) for j, b in enumerate(widths) if b > 0]
                          ) if np.any(np.asarray(widths) > 0) else np.zeros(0, dtype=np.int64)


def calibrate(cfg, H: np.ndarray, W_K: np.ndarray, W_V: np.ndarray, literal: bool = False,
              allocation: str = "waterfill", energy_threshold: float = 0.0) -> dict:
    """Gram -> per (head, side) basis, sigma^2, widths, theta -> W_down / W_up.

    ``cfg`` needs d_model, n_kv_heads, d_head, rank, group, budget_bits,
    count_overhead.  W_down (d_model x N_eff) stacks, for each KV head a and side
    K then V, the columns W V_r of the kept coordinates.  W_up[a][side] is the
    kept rows of V_r^T (n_kept x d_h).
    """
    G = gram(H)
    heads = []
    cols = []
    for a in range(cfg.n_kv_heads):
        sides = {}
        for side, W in (("K", W_K), ("V", W_V)):
            Wa = np.asarray(W, dtype=np.float64)[:, a * cfg.d_head:(a + 1) * cfg.d_head]
            basis = whitened_svd(G, Wa, cfg.rank) if literal else latent_basis(G, Wa, cfg.rank)
            s2 = basis["sigma2"][: cfg.rank]
            n_grp = cfg.rank // cfg.group
            n_elig = n_grp
            if energy_threshold > 0.0:
                re = energy_rank(basis["sigma2"], energy_threshold)  # over all d_head coordinates
                n_elig = min(n_grp, -(-re // cfg.group))
            if allocation == "uniform":
                widths = allocate_widths_uniform(s2, cfg.group, cfg.budget_bits, cfg.count_overhead, n_elig)
            elif allocation == "waterfill":
                widths = np.zeros(n_grp, dtype=np.int64)
                widths[:n_elig] = allocate_widths(s2[: n_elig * cfg.group], cfg.group, cfg.budget_bits,
                                                  cfg.count_overhead)
            else:
                raise ValueError("allocation must be 'waterfill' or 'uniform'")
            payload = int(sum(cfg.group * int(b) for b in widths))
            wf = reverse_water_fill(s2, payload)
            keep = nonzero_coords(widths, cfg.group)
            Vr = basis["V"][:, : cfg.rank]
            sides[side] = dict(V=basis["V"], sigma2=s2, widths=widths, theta=wf["theta"],
                               keep=keep, W_up=Vr[:, keep].T, W_down=(Wa @ Vr)[:, keep])
            cols.append(sides[side]["W_down"])
        heads.append(sides)
    W_down = np.concatenate(cols, axis=1) if cols else np.zeros((cfg.d_model, 0))
    return dict(G=G, heads=heads, W_down=W_down)


# ----------------------------------------------------------------------------
# Per-token quantisation                      [SPECTRA] stage 2/3; fp32 exactness
# ----------------------------------------------------------------------------

def _fp16_sat(x32: np.ndarray) -> np.ndarray:
    return np.clip(np.asarray(x32, dtype=np.float32), np.float32(-FP16_MAX),
                   np.float32(FP16_MAX)).astype(np.float16)


def quantize_groups(x: np.ndarray, b: int, any_width: bool = False):
    """Quantise fp32 latents ``x[..., g]`` (one group per row) to ``b`` bits.

    Every arithmetic step is one IEEE fp32 operation (numpy float32 arithmetic,
    no fused multiply-add): s = fp16((max - min) / (2^b - 1)), z = fp16(min),
    code = clamp(rint((x - z) / s), 0, 2^b - 1), rint rounding half to even;
    s == 0 -> all codes 0.  Returns (codes, s float16, z float16); codes are
    uint8 for the codec's widths {1,2,3,4,8}.  ``any_width`` admits 1..16 bits
    (uint16 codes) for the oracle's own exactness checks.
    """
    if any_width:
        if not 1 <= b <= 16:
            raise ValueError("width must be in 1..16")
    elif b not in (1, 2, 3, 4, 8):
        raise ValueError("width must be one of 1, 2, 3, 4, 8")
    x32 = np.asarray(x, dtype=np.float32)
    mn = x32.min(axis=-1)
    mx = x32.max(axis=-1)
    levels = np.float32(2 ** b - 1)
    s16 = _fp16_sat((mx - mn) / levels)
    z16 = _fp16_sat(mn)
    sf = s16.astype(np.float32)[..., None]
    zf = z16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (x32 - zf) / sf
    codes = np.clip(np.rint(t), np.float32(0), levels)
    codes = np.where(sf > 0, codes, np.float32(0)).astype(np.uint8 if b <= 8 else np.uint16)
    return codes, s16, z16


def dequantize_groups(codes: np.ndarray, s16: np.ndarray, z16: np.ndarray) -> np.ndarray:
    """code * s + z in fp64 (exact for the fp16 scale and zero)."""
    return codes.astype(np.float64) * s16.astype(np.float64)[..., None] \
        + z16.astype(np.float64)[..., None]


def quantize_side(c: np.ndarray, widths, g: int) -> list:
    """Quantise one side's kept latents ``c[T, n_kept]`` group by group.

    Returns a list over the non-empty groups of (b, codes[T, g], s[T], z[T]).
    """
    out = []
    col = 0
    for b in widths:
        b = int(b)
        if b == 0:
            continue
        codes, s, z = quantize_groups(c[:, col:col + g], b)
        out.append((b, codes, s, z))
        col += g
    return out


# ----------------------------------------------------------------------------
# Canonical page layout of the append-only latent cache           [SPECTRA] grouping
# ----------------------------------------------------------------------------
#
# A page holds P tokens of one sequence for every KV head.  Page = head sections
# a = 0..H_kv-1; head section = K section then V section; a side section = for
# each group with b > 0, in ascending group order: its code blocks, then its
# scale/zero records.
#
# Code blocks.  A block holds the codes of 256/g consecutive tokens of one group
# (256 entries, b*32 bytes = 8*b little-endian uint32 words); blocks follow token
# order, P*g/256 of them per page.  Entry (token tau of the block, coordinate k)
# has a fragment position (gid, t4, slot): 32 "lanes" gid*4 + t4 (gid 0..7,
# t4 0..3) with 8 slots each (``fragment_position``).  Its code bit p is stored
# at (word, bit) = ``code_bit_address``:
#   b = 4: word 4*gid + t4, bit 4*slot + p (each lane's 8 codes are one word
#          of nibbles);
#   b = 2: word 2*gid + t4//2, bit 4*slot + 2*(t4 % 2) + p;
#   b = 1: word gid, bit 4*slot + t4;
#   b = 3: bits 0-1 as for b = 2 (words 0..15), bit 2 as for b = 1 in words
#          16 + gid;
#   b = 8: word 2*(4*gid + t4) + (slot // 2) % 2, bit 8*((slot % 2) + 2*(slot // 4)) + p.
#
# Records.  P/2 records of 8 bytes, fp16 {s[2u], s[2u+1], z[2u], z[2u+1]} for the
# token pair u (tokens 2u, 2u+1 of the page).  With 16-token tiles, pair u is
# pair u % 8 of tile u // 8 and sits at record index (u % 8) * (P/16) + u // 8.

def tokens_per_block(g: int) -> int:
    if g not in (8, 16):
        raise ValueError("group must be 8 or 16")
    return 256 // g


def fragment_position(g: int, side: str, tau: int, k: int) -> tuple[int, int, int]:
    """(gid, t4, slot) of entry (token tau in the block, coordinate k in the group)."""
    if g == 16:
        if side == "K":
            row = tau // 2 if tau % 2 == 0 else 8 + tau // 2
            col = k
        else:
            row, col = k, tau
        gid, hh = row % 8, row // 8
        t4, cp, ch = (col % 8) // 2, col % 2, col // 8
        slot = hh + 2 * ch + 4 * cp
    elif g == 8:
        mi, tl = tau // 16, tau % 16
        if side == "K":
            row = tl // 2 if tl % 2 == 0 else 8 + tl // 2
            gid, hh = row % 8, row // 8
            t4, cp = k // 2, k % 2
            slot = hh + 2 * mi + 4 * cp
        else:
            gid = k
            t4, cp, ch = (tl % 8) // 2, tl % 2, tl // 8
            slot = mi + 2 * ch + 4 * cp
    else:
        raise ValueError("group must be 8 or 16")
    return gid, t4, slot


def code_bit_address(g: int, side: str, b: int, tau: int, k: int, p: int) -> tuple[int, int]:
    """(word, bit) inside a block of code bit p of entry (tau, k) of a width-b group."""
    if not 0 <= p < b:
        raise ValueError("bit index out of range")
    gid, t4, slot = fragment_position(g, side, tau, k)
    if b == 4:
        return 4 * gid + t4, 4 * slot + p
    if b == 2 or (b == 3 and p < 2):
        return 2 * gid + t4 // 2, 4 * slot + 2 * (t4 % 2) + p
    if b == 1:
        return gid, 4 * slot + t4
    if b == 3:
        return 16 + gid, 4 * slot + t4
    if b == 8:
        return 2 * (4 * gid + t4) + (slot // 2) % 2, 8 * ((slot % 2) + 2 * (slot // 4)) + p
    raise ValueError("width must be 1, 2, 3, 4 or 8")


def record_index(P: int, tau: int) -> int:
    """Record index of page token tau's pair (see the layout statement above)."""
    u = tau // 2
    return (u % 8) * (P // 16) + u // 8


def _address_table(g: int, side: str, b: int) -> tuple[np.ndarray, np.ndarray]:
    tb = tokens_per_block(g)
    words = np.zeros((b, tb, g), dtype=np.int64)
    bits = np.zeros((b, tb, g), dtype=np.int64)
    for p in range(b):
        for tau in range(tb):
            for k in range(g):
                words[p, tau, k], bits[p, tau, k] = code_bit_address(g, side, b, tau, k, p)
    return words, bits


def side_section_bytes(widths, g: int, P: int) -> int:
    return sum(P * (g * int(b) + 32) // 8 for b in widths if int(b) > 0)


def page_layout(codec_widths, g: int, P: int) -> dict:
    """Byte offsets of every (head, side, kept group) inside a page.

    ``codec_widths[a][side_index]`` is the width vector of head a, side K (0) or
    V (1).  Returns dict(page_bytes, groups) with groups[(a, s)] = list of
    (b, block_offset, record_offset, latent_col) for the non-empty groups.
    """
    if P % 32:
        raise ValueError("page_tokens must be a multiple of 32")
    off = 0
    groups = {}
    for a, per_side in enumerate(codec_widths):
        for s in range(2):
            lst = []
            col = 0
            for b in per_side[s]:
                b = int(b)
                if b == 0:
                    continue
                plane_off = off
                off += b * P * g // 8
                sz_off = off
                off += 4 * P
                lst.append((b, plane_off, sz_off, col))
                col += g
            groups[(a, s)] = lst
    return dict(page_bytes=off, groups=groups)


def pack_group_into_page(page: np.ndarray, g: int, side: str, P: int, b: int,
                         plane_off: int, sz_off: int, tokens: np.ndarray,
                         codes: np.ndarray, s16: np.ndarray, z16: np.ndarray) -> None:
    """Write codes / scale / zero of page-local ``tokens`` into a page (uint8 array).

    Bits of those tokens are cleared first, then set; other tokens are untouched.
    """
    tb = tokens_per_block(g)
    wtab, btab = _address_table(g, side, b)
    words = page[plane_off: plane_off + b * P * g // 8].view("<u4").reshape(P // tb, 8 * b)
    t = np.asarray(tokens, dtype=np.int64)
    blk = np.repeat((t // tb)[:, None], g, axis=1)
    c = np.asarray(codes, dtype=np.uint32)
    for p in range(b):
        w = wtab[p][t % tb]
        bit = btab[p][t % tb].astype(np.uint32)
        one = np.left_shift(np.uint32(1), bit)
        np.bitwise_and.at(words, (blk, w), np.invert(one))
        v = (np.right_shift(c, np.uint32(p)) & np.uint32(1)) << bit
        np.bitwise_or.at(words, (blk, w), v.astype(np.uint32))
    rec = page[sz_off: sz_off + 4 * P].view("<f2").reshape(P // 2, 4)
    ridx = ((t // 2) % 8) * (P // 16) + (t // 2) // 8  # record_index, vectorised
    rec[ridx, t % 2] = np.asarray(s16, dtype=np.float16)
    rec[ridx, 2 + t % 2] = np.asarray(z16, dtype=np.float16)


def unpack_group_from_page(page: np.ndarray, g: int, side: str, P: int, b: int,
                           plane_off: int, sz_off: int, n_tokens: int):
    """Read codes[n_tokens, g], s[n_tokens], z[n_tokens] of a group back from a page."""
    tb = tokens_per_block(g)
    wtab, btab = _address_table(g, side, b)
    words = page[plane_off: plane_off + b * P * g // 8].view("<u4").reshape(P // tb, 8 * b)
    t = np.arange(n_tokens)
    blk, tau = t // tb, t % tb
    codes = np.zeros((n_tokens, g), dtype=np.int64)
    for p in range(b):
        wsel = words[blk[:, None], wtab[p][tau]]
        codes |= ((wsel.astype(np.int64) >> btab[p][tau]) & 1) << p
    rec = page[sz_off: sz_off + 4 * P].view("<f2").reshape(P // 2, 4)
    ridx = ((t // 2) % 8) * (P // 16) + (t // 2) // 8  # record_index, vectorised
    s = rec[ridx, t % 2].astype(np.float16) if n_tokens else np.zeros(0, np.float16)
    z = rec[ridx, 2 + t % 2].astype(np.float16) if n_tokens else np.zeros(0, np.float16)
    return codes.astype(np.uint8), s, z


def append_tokens(pool: np.ndarray, page_bytes: int, layout: dict, codec_widths, g: int, P: int,
                  page_table: np.ndarray, lengths: np.ndarray, seq_ids: np.ndarray,
                  latents: np.ndarray, n_kv: int) -> np.ndarray:
    """Quantise fp32 latents ``latents[T, N_eff]`` and append them to the cache.

    Token i goes to sequence seq_ids[i] at position lengths[seq] + (its rank among
    this call's tokens of that sequence).  Columns of ``latents`` follow W_down:
    head-major, K then V, kept coordinates ascending.  Returns the new lengths.
    """
    lengths = np.array(lengths, dtype=np.int64, copy=True)
    T = latents.shape[0]
    pos = np.zeros(T, dtype=np.int64)
    seen = {}
    for i in range(T):
        sq = int(seq_ids[i])
        pos[i] = lengths[sq] + seen.get(sq, 0)
        seen[sq] = seen.get(sq, 0) + 1
    seqs = np.asarray(seq_ids, dtype=np.int64)
    pg_idx = pos // P
    pids = np.array([int(page_table[seqs[i], pg_idx[i]]) for i in range(T)], dtype=np.int64)
    col0 = 0
    for a in range(n_kv):
        for s, side in enumerate(SIDES):
            widths = codec_widths[a][s]
            nk = sum(g for b in widths if int(b) > 0)
            q = quantize_side(latents[:, col0:col0 + nk].astype(np.float32), widths, g)
            for (b, codes, sc, zr), (b2, plane_off, sz_off, _) in zip(q, layout["groups"][(a, s)]):
                assert b == b2
                for pid in np.unique(pids):
                    sel = np.nonzero(pids == pid)[0]
                    page = pool[pid * page_bytes:(pid + 1) * page_bytes]
                    pack_group_into_page(page, g, side, P, b, plane_off, sz_off,
                                         pos[sel] % P, codes[sel], sc[sel], zr[sel])
            col0 += nk
    for sq, cnt in seen.items():
        lengths[sq] += cnt
    return lengths


def read_side(pool: np.ndarray, page_bytes: int, layout: dict, g: int, P: int,
              page_table_row: np.ndarray, length: int, a: int, s: int) -> np.ndarray:
    """Dequantised kept latents ``[length, n_kept]`` (fp64) of one sequence, head, side."""
    groups = layout["groups"][(a, s)]
    out = np.zeros((length, g * len(groups)))
    n_pages = (length + P - 1) // P
    for pg in range(n_pages):
        pid = int(page_table_row[pg])
        page = pool[pid * page_bytes:(pid + 1) * page_bytes]
        n = min(P, length - pg * P)
        for j, (b, plane_off, sz_off, col) in enumerate(groups):
            side = SIDES[s]
            codes, sc, zr = unpack_group_from_page(page, g, side, P, b, plane_off, sz_off, n)
            out[pg * P: pg * P + n, col:col + g] = dequantize_groups(codes, sc, zr)
    return out


# ----------------------------------------------------------------------------
# Reconstruction and attention            [SPECTRA] stage 3; "Significance" (latent)
# ----------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Exact attention of one query over rows of K, V: softmax(q K^T / sqrt(d)) V, fp64."""
    q = np.asarray(q, dtype=np.float64)
    s = np.asarray(K, dtype=np.float64) @ q / math.sqrt(q.shape[-1])
    m = s.max()
    e = np.exp(s - m)
    return (e / e.sum()) @ np.asarray(V, dtype=np.float64)


def decode_reference(pool: np.ndarray, page_bytes: int, layout: dict, g: int, P: int,
                     page_table: np.ndarray, lengths: np.ndarray, q: np.ndarray,
                     W_up: list, n_q: int, n_kv: int,
                     pairs: list | None = None) -> np.ndarray:
    """Attention over the dequantised cache: rebuild k = c_K W_up^K, v = c_V W_up^V.

    ``q[B, H_q, d_h]`` fp32; ``W_up[a][s]`` (n_kept x d_h).  Returns out[B, H_q,
    d_h] (fp64); with ``pairs`` only those (b, h) entries are filled.
    """
    B = q.shape[0]
    d_h = q.shape[2]
    gq = n_q // n_kv
    out = np.full((B, n_q, d_h), np.nan)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(n_q)]
    cache = {}
    for b, h in todo:
        a = h // gq
        key = (b, a)
        if key not in cache:
            L = int(lengths[b])
            cK = read_side(pool, page_bytes, layout, g, P, page_table[b], L, a, 0)
            cV = read_side(pool, page_bytes, layout, g, P, page_table[b], L, a, 1)
            Kh = cK @ np.asarray(W_up[a][0], dtype=np.float64)
            Vh = cV @ np.asarray(W_up[a][1], dtype=np.float64)
            cache[key] = (Kh, Vh)
        Kh, Vh = cache[key]
        if Kh.shape[0] == 0:
            out[b, h] = 0.0
            continue
        out[b, h] = softmax_attention(q[b, h], Kh, Vh)
    return out


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half form (reading: the pages do not
    model positions; this is the usual form for the models they name): for
    i < d/2 the pair (x_i, x_{i+d/2}) of the row at position p is rotated by the
    angle p * theta^(-2i/d).  ``x[..., n, d]``, ``positions[n]``; fp64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half) / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def decode_reference_rope(pool: np.ndarray, page_bytes: int, layout: dict, g: int, P: int,
                          page_table: np.ndarray, lengths: np.ndarray, q: np.ndarray, W_up: list,
                          n_q: int, n_kv: int, theta: float) -> np.ndarray:
    """Reconstruct-then-attend ([SPECTRA] stage 3): k^, v^ rebuilt from the
    dequantised cache, keys rotated at their positions 0..L-1 and the query at
    position L-1 (theta = 0: no rotation), exact softmax attention."""
    B, d_h = q.shape[0], q.shape[2]
    gq = n_q // n_kv
    out = np.zeros((B, n_q, d_h))
    for b in range(B):
        L = int(lengths[b])
        if L == 0:
            continue
        for a in range(n_kv):
            cK = read_side(pool, page_bytes, layout, g, P, page_table[b], L, a, 0)
            cV = read_side(pool, page_bytes, layout, g, P, page_table[b], L, a, 1)
            Kh = cK @ np.asarray(W_up[a][0], dtype=np.float64)
            Vh = cV @ np.asarray(W_up[a][1], dtype=np.float64)
            if theta > 0:
                Kh = rope(Kh, np.arange(L), theta)
            for h in range(a * gq, (a + 1) * gq):
                qh = np.asarray(q[b, h], dtype=np.float64)[None, :]
                if theta > 0:
                    qh = rope(qh, np.array([L - 1]), theta)
                out[b, h] = softmax_attention(qh[0], Kh, Vh)
    return out


# ----------------------------------------------------------------------------
# W_O correction                                   [SPECTRA] stage 1, "Refinement"
# ----------------------------------------------------------------------------

def causal_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    n, d = Q.shape
    s = (Q @ K.T) / math.sqrt(d)
    s = np.where(np.tril(np.ones((n, n), dtype=bool)), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ V


def wo_correction(H: np.ndarray, W_Q: np.ndarray, W_K: np.ndarray, W_V: np.ndarray,
                  W_O: np.ndarray, codec: dict, n_q: int, n_kv: int, d_h: int,
                  eps_rel: float = 1e-8) -> dict:
    """Closed-form, training-free W_O correction (parity unpinned beyond special cases).

    Reading: for each q head h (KV head a = h // Gq), on the calibration tokens as
    one causal sequence, O_h is the attention output with exact K, V and O^_h the
    one with the rank-truncated, unquantised K, V (kept coordinates only:
    k~ = k V_r P V_r^T).  O^_h lies in the span of the kept value directions U_a,
    so write O^_h = L_h U_a^T (L_h = latent output).  The least-squares map from
    L_h to O_h, M'_h = (L_h^T L_h + eps I)^-1 L_h^T O_h with eps = eps_rel
    tr(L_h^T L_h)/n_kept, gives M_h = U_a M'_h and W_O' = blockdiag(M_h) W_O.
    As eps -> 0 this is the minimum-norm solution of min ||O^_h M - O_h||.  Pinned
    only by: M_h = I when nothing is truncated (eps -> 0), and the corrected
    residual never exceeds the uncorrected one.
    """
    H64 = np.asarray(H, dtype=np.float64)
    gq = n_q // n_kv
    W_O = np.asarray(W_O, dtype=np.float64)
    W_Op = np.array(W_O, copy=True)
    Ms = []
    for h in range(n_q):
        a = h // gq
        sl = slice(a * d_h, (a + 1) * d_h)
        q = H64 @ np.asarray(W_Q, dtype=np.float64)[:, h * d_h:(h + 1) * d_h]
        k = H64 @ np.asarray(W_K, dtype=np.float64)[:, sl]
        v = H64 @ np.asarray(W_V, dtype=np.float64)[:, sl]
        hk, hv = codec["heads"][a]["K"], codec["heads"][a]["V"]
        Vk = hk["V"][:, hk["keep"]]
        U = hv["V"][:, hv["keep"]]
        O = causal_attention(q, k, v)
        lat = causal_attention(q, k @ Vk @ Vk.T, v @ U)  # latent value output L_h
        if U.shape[1] == 0:
            M = np.zeros((d_h, d_h))
        else:
            A = lat.T @ lat
            eps = eps_rel * np.trace(A) / U.shape[1]
            Mp = np.linalg.solve(A + eps * np.eye(U.shape[1]), lat.T @ O)
            M = U @ Mp
        Ms.append(M)
        W_Op[h * d_h:(h + 1) * d_h, :] = M @ W_O[h * d_h:(h + 1) * d_h, :]
    return dict(M=Ms, W_O=W_Op)
