"""Plain CPU oracle of the FlashLoop lazy loop-r attention sublayer.

TEST INFRASTRUCTURE.  Only the test-suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The CUDA
library never calls it and shares no code with it.

Sources (cited by page title and section):
  [FL] "FlashLoop: Fast and Memory-Efficient Looped Transformers via Lazy
       Updates" (Yang & Liu), digest of §3.1-§4.4, App. D.1-D.3, App. E, App. G.
  [FZ] "FlashLoop, or: Looping a Transformer Quadruples the Bill and Then
       Throws Most of It Away", §1 (Cell 1) and §3 (Cell 3).
  [SK] "Flashloop Lazy Updates" skill card, Method §1-§3.

Precision.  Projections, RoPE and attention run in float64 on the exact
values of the bf16 inputs.  Values the method stores in bf16 (q, the
attention output O, the projection Y) are rounded to bf16 when stored.
The quantiser takes its integer decisions in float32 with IEEE division and
round-half-even, the same precision the kernel uses, so codes agree bit for
bit on identical float32 residuals.  The gate compares squared norms in
float64.

Readings where the pages leave a step open (each the plainest one the rest
supports):
  R1 gate: a token stays active iff ||X_r - X_{r-1}||^2 >= tau^2 ||X_{r-1}||^2,
     candidates are the previous active set, so the sets nest [FL §4.1, D.1].
  R2 the removed "old" contribution of pair (i, j) at loop r is the one
     counted at loop r-1: score q_i^(r-1) . Khat_j^(r-1), value Vhat_j^(r-1)
     [FL §4.2, D.2]; nesting of rows and columns makes this well defined.
  R3 the running state (m, N, Z) plays the role of the cached global mass:
     unselected columns keep their counted contribution [FL §4.2].
  R4 every attention read uses the reconstructed (dequantised) KV, loop 1
     included [FL App. G].
  R5 residuals are taken against the reconstructed previous loop, and only
     active tokens store one [FL §4.3, D.3].
  R6 quantiser: symmetric, groups of 32 along head_dim, qmax = 2^(b-1)-1,
     s = fp16(max|x| / qmax), code = clamp(rint(x / s)), s = 0 -> codes 0.
  R7 RoPE rotate-half, pairs (d, d + dh/2), position = token index, theta 1e4.
  R8 top-k ranks by value descending, ties to the lower index; returned
     ascending.  For r >= 3 the candidates are the previous selection.
  R9 column mass at loop 1 is the dense column sum of the softmax; at r >= 2
     it is summed over active rows for the selected columns only.
  R10 fixed-mass form (the pages' eq. 3 reading, an option): each row's
     selected columns J keep the total probability M_i they had in the
     previous loop's full distribution; within J the mass is shared in
     proportion to e^(s_new).  Unselected columns keep their probabilities,
     so every row's distribution still sums to one [FL §4.2, D.2; FZ §3].
  R11 the pages' own cache setting (an option): INT4 asymmetric groups of
     64 with an fp16 scale and an fp16 minimum, keys grouped per channel over
     64 tokens (residual keys over 64 entries of the loop's active list),
     values per token over 64 channels, the last 64 tokens in bf16 at every
     loop [FL App. E; FZ §3].

Parity unpinned: nothing in this module is without a pin; the accuracy and
reconstruction figures the paper reports on real models are out of reach
(they need trained weights and datasets).
"""
from __future__ import annotations

import math

import numpy as np

from workload.gen import bf16_bits_to_f32, f32_to_bf16_bits

QMAX = {8: 127, 4: 7, 2: 1}
GROUP = 32


# --------------------------------------------------------------------------
# small helpers
# --------------------------------------------------------------------------
def bf16_vals(bits) -> np.ndarray:
    """float64 values of bf16 bit patterns."""
    return bf16_bits_to_f32(bits).astype(np.float64)


def to_bf16_bits(x) -> np.ndarray:
    """Store a float64 result as bf16: round to float32, then to bf16."""
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


# --------------------------------------------------------------------------
# (a1) token change gate and compaction  [FL §3.1, §4.1, App. D.1; SK Method §1]
# --------------------------------------------------------------------------
def gate_norms(x_cur_bits, x_prev_bits, candidates):
    """Squared change D_i and squared previous norm P_i for candidate rows (float64)."""
    xc = bf16_vals(x_cur_bits[candidates])
    xp = bf16_vals(x_prev_bits[candidates])
    diff = xc - xp
    return (diff * diff).sum(axis=1), (xp * xp).sum(axis=1)


def gate(x_cur_bits, x_prev_bits, candidates, tau):
    """Active set A^(r): candidates whose relative L2 change reaches tau (reading R1).

    ``candidates`` is the ascending previous active set; the result keeps
    that order (a stable compaction).
    """
    candidates = np.asarray(candidates, dtype=np.int64)
    D, P = gate_norms(x_cur_bits, x_prev_bits, candidates)
    keep = D >= (tau * tau) * P
    return candidates[keep]


def gate_topk(x_cur_bits, x_prev_bits, candidates, budget):
    """Active set A^(r) by top-k token retention [FL §4.1, App. D.1]: the
    ``budget`` candidates of largest normalised change ||x_r - x_(r-1)||^2 /
    ||x_(r-1)||^2 (the square ranks like the norm ratio), ties to the lower
    token, returned ascending.  A zero previous row ranks first if it changed
    and last if it did not.  Keys are ranked in float32, as a float32 kernel
    would hold them.
    """
    candidates = np.asarray(candidates, dtype=np.int64)
    if budget >= candidates.size:
        return candidates
    D, P = gate_norms(x_cur_bits, x_prev_bits, candidates)
    with np.errstate(divide="ignore", invalid="ignore"):
        key = np.where(P > 0, D / np.where(P > 0, P, 1.0), np.where(D > 0, np.inf, 0.0))
    dense = np.full(int(candidates.max()) + 1, -np.inf, dtype=np.float32)
    dense[candidates] = key.astype(np.float32)
    return topk_columns(dense, candidates, budget)


# --------------------------------------------------------------------------
# (a2) projections and RoPE  [FL §4.3 "post-RoPE keys", App. E; App. G]
# --------------------------------------------------------------------------
def rope_angles(positions, head_dim, theta):
    """Angle p * theta^(-2t/dh) for t < dh/2 (float64)."""
    half = head_dim // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / head_dim)
    return np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]


def apply_rope(x, positions, theta):
    """Rotate-half RoPE on x [n, H, dh] at the given token positions (reading R7)."""
    dh = x.shape[-1]
    half = dh // 2
    ang = rope_angles(positions, dh, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def head_rows(w_bits, heads, head_dim):
    """Rows of an [out, in] weight that produce the given heads' outputs."""
    idx = np.concatenate([np.arange(h * head_dim, (h + 1) * head_dim) for h in heads])
    return w_bits[idx]


def project_qkv(x_rows_bits, positions, W, heads, head_dim, theta):
    """q, k, v for the given rows and heads: x W^T, RoPE on q and k (float64).

    Returns q rounded to bf16 (it is stored), k and v in float64.
    """
    x = bf16_vals(x_rows_bits)
    n = x.shape[0]
    out = []
    for name in ("wq", "wk", "wv"):
        w = bf16_vals(head_rows(W[name], heads, head_dim))
        out.append((x @ w.T).reshape(n, len(heads), head_dim))
    q, k, v = out
    q = apply_rope(q, positions, theta)
    k = apply_rope(k, positions, theta)
    return to_bf16_bits(q), k, v


# --------------------------------------------------------------------------
# (a3) group quantiser and packing  [FL §3.3, §4.3, App. D.3; reading R6]
# --------------------------------------------------------------------------
def quantize_groups(x32, bits):
    """Symmetric group quantisation of float32 x [..., dh] in groups of 32.

    Returns (codes int8 [..., dh], scales float16 [..., dh/32]).  Every
    decision is a float32 operation: max|x|, the division by qmax, the
    rounding to fp16, the division x / s and round-half-even.
    """
    qmax = QMAX[bits]
    x32 = np.asarray(x32, dtype=np.float32)
    g = x32.reshape(x32.shape[:-1] + (x32.shape[-1] // GROUP, GROUP))
    amax = np.max(np.abs(g), axis=-1)
    with np.errstate(over="ignore"):
        s16 = (amax / np.float32(qmax)).astype(np.float16)
    s16 = np.minimum(s16, np.float16(65504.0))
    s32 = s16.astype(np.float32)[..., None]
    q = np.zeros_like(g)
    np.divide(g, s32, out=q, where=np.broadcast_to(s32 > 0, g.shape))
    codes = np.clip(np.rint(q), -qmax, qmax).astype(np.int8)
    return codes.reshape(x32.shape), s16


def dequantize_groups(codes, s16):
    """code * scale in float32 (exact: both factors are short)."""
    c = np.asarray(codes).astype(np.float32)
    g = c.reshape(c.shape[:-1] + (c.shape[-1] // GROUP, GROUP))
    return (g * s16.astype(np.float32)[..., None]).reshape(c.shape)


def pack_codes(codes, bits):
    """Bit-pack two's-complement codes along the last axis.

    INT8: one byte each.  INT4: element 2t in the low nibble of byte t,
    2t+1 in the high nibble.  INT2: element 4t+u in bits [2u, 2u+1] of byte t.
    """
    c = np.asarray(codes).astype(np.int64)
    if bits == 8:
        return (c & 0xFF).astype(np.uint8)
    per = 8 // bits
    mask = (1 << bits) - 1
    c = (c & mask).reshape(c.shape[:-1] + (c.shape[-1] // per, per))
    out = np.zeros(c.shape[:-1], dtype=np.int64)
    for u in range(per):
        out |= c[..., u] << (bits * u)
    return out.astype(np.uint8)


def unpack_codes(packed, bits):
    """Inverse of pack_codes: int8 codes, sign-extended."""
    p = np.asarray(packed).astype(np.int64)
    if bits == 8:
        return p.astype(np.uint8).view(np.int8).astype(np.int8)
    per = 8 // bits
    mask = (1 << bits) - 1
    fields = [(p >> (bits * u)) & mask for u in range(per)]
    f = np.stack(fields, axis=-1)
    f = np.where(f >= (1 << (bits - 1)), f - (1 << bits), f)
    return f.reshape(p.shape[:-1] + (p.shape[-1] * per,)).astype(np.int8)


class KVStream:
    """One of the K or V caches of a sequence: a quantised loop-1 base plus
    per-loop residual streams for active tokens only [FL §4.3, App. D.3].

    ``tokens`` = token count, ``heads`` = number of heads held.  With
    ``quantize=False`` the same bookkeeping stores exact float64 values (used
    to pin the attention algebra against textbook attention).
    """

    def __init__(self, tokens, heads, head_dim, bits_per_loop, quantize=True):
        self.T, self.H, self.dh = tokens, heads, head_dim
        self.bits = list(bits_per_loop)
        self.quantize = quantize
        self.base = None          # (codes, scales) or float64 values
        self.res = {}             # loop -> (codes, scales) or float64 values, compact rows
        self.slot = {}            # loop -> int64 [tokens], -1 when the token is absent

    # -- loop 1 -------------------------------------------------------------
    def write_base(self, x):
        """Quantise the loop-1 values of every token (INT8 base)."""
        if self.quantize:
            self.base = quantize_groups(np.asarray(x).astype(np.float32), self.bits[0])
        else:
            self.base = np.asarray(x, dtype=np.float64).copy()

    def _deq(self, item, rows):
        if self.quantize:
            codes, s16 = item
            return dequantize_groups(codes[rows], s16[rows])
        return item[rows]

    # -- reconstruction -----------------------------------------------------
    def reconstruct(self, tokens, loop):
        """Xhat^(loop) for the given tokens: base plus, in loop order, the
        residual of every loop 2..loop where the token was active (float32
        additions in that order; float64 when not quantising)."""
        tokens = np.asarray(tokens, dtype=np.int64)
        acc = self._deq(self.base, tokens)
        for l in range(2, loop + 1):
            if l not in self.slot:
                continue
            sl = self.slot[l][tokens]
            have = sl >= 0
            if not np.any(have):
                continue
            add = np.zeros_like(acc)
            add[have] = self._deq(self.res[l], sl[have])
            acc = acc + add
        return acc

    # -- loops r >= 2 -------------------------------------------------------
    def write_residual(self, loop, tokens, x):
        """Store the quantised residual x - Xhat^(loop-1) for the active tokens
        (reading R5); tokens are the ascending active set, slot = position."""
        tokens = np.asarray(tokens, dtype=np.int64)
        prev = self.reconstruct(tokens, loop - 1)
        if self.quantize:
            rho = np.asarray(x).astype(np.float32) - prev
            self.res[loop] = quantize_groups(rho, self.bits[loop - 1])
        else:
            self.res[loop] = np.asarray(x, dtype=np.float64) - prev
        slot = np.full(self.T, -1, dtype=np.int64)
        slot[tokens] = np.arange(tokens.size)
        self.slot[loop] = slot

    def residual_codes(self, loop):
        return self.res[loop][0]

    def residual_scales(self, loop):
        return self.res[loop][1]


# --------------------------------------------------------------------------
# (f2) the pages' own cache setting  [FL App. E "Quantization Setting"; FZ §3]
# --------------------------------------------------------------------------
PAPER_GROUP = 64
PAPER_TAIL = 64
PAPER_LEVELS = 15          # INT4 asymmetric: codes 0..15


def quantize_asym(g32):
    """Asymmetric INT4 quantisation of float32 groups along the last axis
    (reading R11).  Per group: lo = fp16(min), s = fp16((max - min) / 15),
    code = clamp(rint((x - lo) / s), 0, 15) in float32 with IEEE division and
    round-half-even; s = 0 gives code 0.  Returns (codes uint8, s fp16, lo fp16)."""
    g32 = np.asarray(g32, dtype=np.float32)
    mn = np.min(g32, axis=-1)
    mx = np.max(g32, axis=-1)
    with np.errstate(over="ignore"):
        lo16 = mn.astype(np.float16)
        s16 = ((mx - mn) / np.float32(PAPER_LEVELS)).astype(np.float16)
    s32 = s16.astype(np.float32)[..., None]
    q = np.zeros_like(g32)
    np.divide(g32 - lo16.astype(np.float32)[..., None], s32, out=q, where=np.broadcast_to(s32 > 0, g32.shape))
    codes = np.clip(np.rint(q), 0, PAPER_LEVELS).astype(np.uint8)
    return codes, s16, lo16


def dequantize_asym(codes, s16, lo16):
    """code * s + lo in float32."""
    return (np.asarray(codes).astype(np.float32) * s16.astype(np.float32)[..., None]
            + lo16.astype(np.float32)[..., None])


class PaperKVStream:
    """One of K or V in the pages' own setting (reading R11): an INT4
    asymmetric base over the tokens before the last 64, groups of 64 along
    the token axis per channel for keys and along the channels per token for
    values, residuals of later loops in the same format for the active
    tokens (key groups run over 64 consecutive entries of the loop's active
    list), and the last 64 tokens kept in bf16 at every loop they are active.
    Same interface as KVStream."""

    def __init__(self, tokens, heads, head_dim, kind, tail=PAPER_TAIL, group=PAPER_GROUP):
        assert kind in ("k", "v") and head_dim % group == 0
        self.T, self.H, self.dh = tokens, heads, head_dim
        self.kind, self.tail, self.group = kind, min(tail, tokens), group
        self.body = tokens - self.tail       # tokens [0, body) are quantised
        self.base = None                     # (codes, s, lo) of the body
        self.res = {}                        # loop -> (codes, s, lo, n) of the active body tokens
        self.tail_vals = {}                  # loop -> (tokens, bf16 bits [n, H, dh]) of the active tail tokens
        self.slot = {}                       # loop -> int64 [tokens], -1 when absent (body tokens only)
        self.active = {}                     # loop -> ascending active tokens

    # -- group layout ---------------------------------------------------------
    def _quant(self, x):
        """x float32 [n, H, dh] -> quantised groups (codes, s, lo, n)."""
        n = x.shape[0]
        G = self.group
        if self.kind == "v":                       # per token: groups of G channels
            g = x.reshape(n, self.H, self.dh // G, G)
            return quantize_asym(g) + (n,)
        pad = (-n) % G                              # per channel: groups of G rows
        xp = np.concatenate([x, np.repeat(x[-1:], pad, axis=0)]) if pad and n else x
        g = xp.reshape(-1, G, self.H, self.dh).transpose(0, 2, 3, 1)   # [groups, H, dh, G]
        codes, s16, lo16 = quantize_asym(g)
        return codes, s16, lo16, n

    def _deq(self, item, rows):
        codes, s16, lo16, n = item
        rows = np.asarray(rows, dtype=np.int64)
        if self.kind == "v":
            return dequantize_asym(codes[rows], s16[rows], lo16[rows]).reshape(rows.size, self.H, self.dh)
        G = self.group
        grp, off = rows // G, rows % G
        c = codes[grp, :, :, off]                                        # [r, H, dh]: row `off` of group `grp`
        return c.astype(np.float32) * s16[grp].astype(np.float32) + lo16[grp].astype(np.float32)

    # -- loop 1 ---------------------------------------------------------------
    def write_base(self, x):
        x = np.asarray(x)
        self.base = self._quant(x[: self.body].astype(np.float32))
        toks = np.arange(self.body, self.T)
        self.tail_vals[1] = (toks, to_bf16_bits(x[self.body:]))
        self.active[1] = np.arange(self.T)

    def _tail_value(self, tok, loop):
        for l in range(loop, 0, -1):
            if l in self.tail_vals:
                toks, bits = self.tail_vals[l]
                i = np.searchsorted(toks, tok)
                if i < toks.size and toks[i] == tok:
                    return bf16_vals(bits[i])
        raise KeyError(tok)

    # -- reconstruction -------------------------------------------------------
    def reconstruct(self, tokens, loop):
        """Xhat^(loop): for body tokens the base plus every residual of loops
        2..loop where the token was active (float32, loop order); for tail
        tokens the bf16 value of the latest loop <= `loop` that stored one."""
        tokens = np.asarray(tokens, dtype=np.int64)
        out = np.zeros((tokens.size, self.H, self.dh), dtype=np.float64)
        body = tokens < self.body
        if np.any(body):
            bt = tokens[body]
            acc = self._deq(self.base, bt)
            for l in range(2, loop + 1):
                if l not in self.slot:
                    continue
                sl = self.slot[l][bt]
                have = sl >= 0
                if np.any(have):
                    add = np.zeros_like(acc)
                    add[have] = self._deq(self.res[l], sl[have])
                    acc = acc + add
            out[body] = acc
        for i in np.nonzero(~body)[0]:
            out[i] = self._tail_value(int(tokens[i]), loop)
        return out

    # -- loops r >= 2 ---------------------------------------------------------
    def write_residual(self, loop, tokens, x):
        """Body tokens store the quantised x - Xhat^(loop-1); tail tokens store
        x in bf16.  ``tokens`` ascending, x [n, H, dh]."""
        tokens = np.asarray(tokens, dtype=np.int64)
        x = np.asarray(x)
        body = tokens < self.body
        bt = tokens[body]
        rho = x[body].astype(np.float32) - self.reconstruct(bt, loop - 1).astype(np.float32)
        self.res[loop] = self._quant(rho)
        slot = np.full(self.T, -1, dtype=np.int64)
        slot[bt] = np.arange(bt.size)
        self.slot[loop] = slot
        self.tail_vals[loop] = (tokens[~body], to_bf16_bits(x[~body]))
        self.active[loop] = tokens

    def stored_bytes(self):
        """Bytes of everything stored: 4-bit codes, an fp16 scale and an fp16
        minimum per group, bf16 tail values."""
        def q_bytes(item):
            codes, s16, lo16, n = item
            if self.kind == "v":
                elems = n * self.H * self.dh
            else:   # the padding rows of a partial key group store no codes
                elems = n * self.H * self.dh
            return elems // 2 + 2 * s16.size + 2 * lo16.size
        total = q_bytes(self.base)
        for item in self.res.values():
            total += q_bytes(item)
        for toks, _ in self.tail_vals.values():
            total += toks.size * self.H * self.dh * 2
        return total


def paper_cache_bytes(S, n_heads, head_dim, body_active, tail_active, tail=PAPER_TAIL, group=PAPER_GROUP):
    """Bytes of K and V in the pages' own setting (reading R11), by formula:
    the body's 4-bit codes plus 4 bytes (fp16 scale and minimum) per group of
    64, and 2 bytes per element of the bf16 tail at every loop it is stored.
    ``body_active[l]`` / ``tail_active[l]`` = active body / tail tokens of loop
    l+1 (index 0: loop 1, every token)."""
    E = n_heads * head_dim
    total = 0
    for l, (nb, nt) in enumerate(zip(body_active, tail_active)):
        codes = 2 * nb * E // 2
        v_groups = nb * E // group
        k_groups = -(-nb // group) * E
        total += codes + 4 * (v_groups + k_groups) + 2 * nt * E * 2
    return total


# --------------------------------------------------------------------------
# (a4) column selection  [FL §3.2, §4.2, App. D.2; FZ §3; reading R8]
# --------------------------------------------------------------------------
def topk_columns(mass32, candidates, k):
    """k columns of largest float32 mass among the candidates, ties to the
    lower index, returned in ascending index order."""
    candidates = np.asarray(candidates, dtype=np.int64)
    vals = np.asarray(mass32, dtype=np.float32)[candidates].astype(np.float64)
    vals = vals + 0.0  # -0 and +0 compare equal
    order = np.lexsort((candidates, -vals))
    return np.sort(candidates[order[:k]])


# --------------------------------------------------------------------------
# (a6) attention  [FL §3.2, §4.2, App. D.2, App. G; FZ §3; readings R2-R4, R9]
# --------------------------------------------------------------------------
def dense_causal_attention(q_bits, Khat, Vhat, row_chunk=512):
    """Loop 1 of one head: for every row i the running state over j <= i.

    m_i = max_j s_ij, Z_i = sum_j e^(s_ij - m_i), N_i = sum_j e^(s_ij - m_i) Vhat_j,
    s_ij = q_i . Khat_j / sqrt(dh); and the column mass
    c[j] = sum_{i >= j} e^(s_ij - m_i) / Z_i.  Rows are independent; they are
    processed in chunks only to bound memory.
    """
    q = bf16_vals(q_bits)
    S, dh = q.shape
    Kt = np.asarray(Khat, dtype=np.float64).T
    V = np.asarray(Vhat, dtype=np.float64)
    scale = 1.0 / math.sqrt(dh)
    m = np.empty(S)
    Z = np.empty(S)
    N = np.empty((S, dh))
    c = np.zeros(S)
    cols = np.arange(S)
    for i0 in range(0, S, row_chunk):
        i1 = min(S, i0 + row_chunk)
        rows = np.arange(i0, i1)
        s = (q[i0:i1] @ Kt[:, :i1]) * scale
        valid = cols[None, :i1] <= rows[:, None]
        s = np.where(valid, s, -np.inf)
        mi = s.max(axis=1)
        e = np.exp(s - mi[:, None])
        Zi = e.sum(axis=1)
        m[i0:i1], Z[i0:i1] = mi, Zi
        N[i0:i1] = e @ V[:i1]
        c[:i1] += (e / Zi[:, None]).sum(axis=0)
    return m, Z, N, c


def sparse_update(rows, T, q_old_bits, q_new_bits, K_old, K_new, V_old, V_new, m, Z, N,
                  row_chunk=2048):
    """Loop r >= 2 of one head: replace, for every active row i and selected
    column j <= i, the loop r-1 contribution by the loop r one.

      s_old = q_i^(r-1) . Khat_j^(r-1) / sqrt(dh),  s_new = q_i^(r) . Khat_j^(r) / sqrt(dh)
      m'  = max(m_i, max_J s_new),  a = e^(m_i - m')
      Z'  = a Z_i - sum_J e^(s_old - m') + sum_J e^(s_new - m')
      N'  = a N_i - sum_J e^(s_old - m') Vhat_j^(r-1) + sum_J e^(s_new - m') Vhat_j^(r)

    ``rows`` ascending active tokens, ``T`` ascending selected columns;
    K_*/V_* are the reconstructed columns of T [k, dh].  Returns (m', Z', N')
    for the rows and the column mass sum_i e^(s_new - m') / Z' over T.
    """
    rows = np.asarray(rows, dtype=np.int64)
    T = np.asarray(T, dtype=np.int64)
    dh = K_old.shape[1]
    scale = 1.0 / math.sqrt(dh)
    qo = bf16_vals(q_old_bits)
    qn = bf16_vals(q_new_bits)
    Ko_t = np.asarray(K_old, dtype=np.float64).T
    Kn_t = np.asarray(K_new, dtype=np.float64).T
    Vo = np.asarray(V_old, dtype=np.float64)
    Vn = np.asarray(V_new, dtype=np.float64)
    m2 = np.empty(rows.size)
    Z2 = np.empty(rows.size)
    N2 = np.empty((rows.size, dh))
    cmass = np.zeros(T.size)
    for a0 in range(0, rows.size, row_chunk):
        a1 = min(rows.size, a0 + row_chunk)
        valid = T[None, :] <= rows[a0:a1, None]
        s_old = (qo[a0:a1] @ Ko_t) * scale
        s_new = (qn[a0:a1] @ Kn_t) * scale
        smax = np.where(valid, s_new, -np.inf).max(axis=1) if T.size else np.full(a1 - a0, -np.inf)
        mi = np.asarray(m[a0:a1], dtype=np.float64)
        mn = np.maximum(mi, smax)
        alpha = np.exp(mi - mn)
        e_old = np.where(valid, np.exp(s_old - mn[:, None]), 0.0)
        e_new = np.where(valid, np.exp(s_new - mn[:, None]), 0.0)
        Zn = alpha * Z[a0:a1] - e_old.sum(axis=1) + e_new.sum(axis=1)
        Nn = alpha[:, None] * N[a0:a1] - e_old @ Vo + e_new @ Vn
        m2[a0:a1], Z2[a0:a1], N2[a0:a1] = mn, Zn, Nn
        cmass += (e_new / Zn[:, None]).sum(axis=0)
    return m2, Z2, N2, cmass


def dense_causal_probs(q_bits, Khat):
    """The full causal softmax of one head as an explicit [S, S] matrix:
    P[i, j] = e^(s_ij) / sum_{j' <= i} e^(s_ij') for j <= i, 0 above the
    diagonal (s_ij = q_i . Khat_j / sqrt(dh))."""
    q = bf16_vals(q_bits)
    S, dh = q.shape
    s = (q @ np.asarray(Khat, dtype=np.float64).T) / math.sqrt(dh)
    s = np.where(np.tri(S, dtype=bool), s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def fixed_mass_update(rows, T, q_new_bits, K_new, V_old, V_new, P, O):
    """Loop r >= 2 of one head in the fixed-mass form (reading R10), on the
    explicit distributions.  For every active row i with J = {j in T : j <= i}:

      M_i = sum_J P[i, j]                             (cached mass of the selection)
      P'[i, j] = M_i e^(s_new_ij) / sum_J e^(s_new)    for j in J, else P[i, j]
      O'_i = O_i - sum_J P[i, j] Vhat_j^(r-1) + sum_J P'[i, j] Vhat_j^(r)

    P [S, S] and O [S, dh] (float64) are updated in place; returns the column
    mass sum_i P'[i, j] over the active rows for j in T."""
    rows = np.asarray(rows, dtype=np.int64)
    T = np.asarray(T, dtype=np.int64)
    dh = K_new.shape[1]
    qn = bf16_vals(q_new_bits)
    s_new = (qn @ np.asarray(K_new, dtype=np.float64).T) / math.sqrt(dh)   # [n, k]
    Vo = np.asarray(V_old, dtype=np.float64)
    Vn = np.asarray(V_new, dtype=np.float64)
    cmass = np.zeros(T.size)
    for a, i in enumerate(rows):
        sel = T <= i
        if not sel.any():
            continue
        J = T[sel]
        p_old = P[i, J].copy()
        M = p_old.sum()
        e = np.exp(s_new[a, sel] - s_new[a, sel].max())
        p_new = M * e / e.sum()
        O[i] = O[i] - p_old @ Vo[sel] + p_new @ Vn[sel]
        P[i, J] = p_new
        cmass[sel] += p_new
    return cmass


def out_projection(o_bits, wo_bits):
    """Y = O W_o^T for the given rows, stored as bf16 (float64 arithmetic)."""
    return to_bf16_bits(bf16_vals(o_bits) @ bf16_vals(wo_bits).T)


# --------------------------------------------------------------------------
# one prefill sequence, loops 1..R  [FL §4, App. D]
# --------------------------------------------------------------------------
class OracleSequence:
    """Runs the sublayer over loops 1..R for one sequence.

    ``heads`` restricts the per-head work (projections, caches, attention) to
    a subset; the output projection Y needs every head and is computed only
    when all heads are held.  ``topk`` overrides the per-loop column budget
    (index r-1), ``tau`` the gate threshold, ``quantize=False`` keeps exact KV.
    """

    def __init__(self, cfg, W, X, heads=None, quantize=True, topk=None, tau=None,
                 keep_history=True, token_budgets=None, fixed_mass=False, kv_scheme="spec"):
        """``token_budgets`` (per loop, index r-1) switches the gate from the
        tau threshold to top-k token retention with those budgets.
        ``fixed_mass`` runs loops >= 2 in the fixed-mass form (reading R10)
        on explicit [S, S] distributions per head (small S only).
        ``kv_scheme="paper"`` stores K and V in the pages' own setting
        (reading R11) instead of the INT8 + INT4/INT2 symmetric streams."""
        self.cfg = cfg
        self.fixed_mass = fixed_mass
        self.P = None          # fixed-mass form: head -> [S, S] probabilities
        self.Ofm = None        # fixed-mass form: head -> [S, dh] float64 outputs
        self.token_budgets = None if token_budgets is None else list(token_budgets)
        self.W = W
        self.X = X
        self.S = cfg.seq
        self.dh = cfg.head_dim
        self.heads = list(range(cfg.n_heads)) if heads is None else list(heads)
        self.all_heads = len(self.heads) == cfg.n_heads
        self.tau = cfg.tau if tau is None else tau
        self.kbud = list(cfg.k_per_loop() if topk is None else topk)
        self.keep = keep_history
        Hs = len(self.heads)
        if kv_scheme == "paper":
            self.Kc = PaperKVStream(self.S, Hs, self.dh, "k")
            self.Vc = PaperKVStream(self.S, Hs, self.dh, "v")
        else:
            self.Kc = KVStream(self.S, Hs, self.dh, cfg.bits, quantize)
            self.Vc = KVStream(self.S, Hs, self.dh, cfg.bits, quantize)
        self.active = {}
        self.q = {}            # loop -> bf16 bits [S, Hs, dh] (rows active at that loop set)
        self.k_exact = {}      # loop -> float64 [n, Hs, dh] of the active rows
        self.v_exact = {}
        self.T = {}            # loop -> list over held heads of ascending columns
        self.colmass = {}      # loop -> float64 [Hs, S]
        self.m = self.Z = self.N = None
        self.hist = {}         # loop -> (m, Z, N) copies
        self.O = np.zeros((self.S, Hs * self.dh), dtype=np.uint16)
        self.Y = np.zeros((self.S, cfg.d_model), dtype=np.uint16) if self.all_heads else None
        self.O_hist = {}
        self.Y_hist = {}
        self.loop = 0

    # ------------------------------------------------------------------
    def _project(self, r, rows):
        q, k, v = project_qkv(self.X[r - 1][rows], rows, self.W, self.heads, self.dh,
                              self.cfg.rope_theta)
        qfull = self.q.get(r - 1)
        qfull = np.zeros((self.S, len(self.heads), self.dh), np.uint16) if qfull is None else qfull.copy()
        qfull[rows] = q
        self.q[r] = qfull
        self.k_exact[r], self.v_exact[r] = k, v
        return k, v

    def _store_output(self, r, rows):
        Hs, dh = len(self.heads), self.dh
        if self.fixed_mass:
            O = self.Ofm[:, rows, :]
        else:
            O = self.N[:, rows, :] / self.Z[:, rows, None]        # [Hs, n, dh]
        self.O[rows] = to_bf16_bits(O.transpose(1, 0, 2).reshape(rows.size, Hs * dh))
        if self.all_heads:
            self.Y[rows] = out_projection(self.O[rows], self.W["wo"])
        if self.keep:
            self.hist[r] = (self.m.copy(), self.Z.copy(), self.N.copy())
            self.O_hist[r] = self.O.copy()
            if self.all_heads:
                self.Y_hist[r] = self.Y.copy()

    def run_loop1(self):
        """Dense loop: every token, INT8 base, dense causal attention on the
        reconstructed base, column mass c^(1) [FL App. D.1: the early loops run dense]."""
        S, dh = self.S, self.dh
        rows = np.arange(S)
        self.active[1] = rows
        k, v = self._project(1, rows)
        self.Kc.write_base(k)
        self.Vc.write_base(v)
        Kh = self.Kc.reconstruct(rows, 1)
        Vh = self.Vc.reconstruct(rows, 1)
        Hs = len(self.heads)
        self.m = np.empty((Hs, S)); self.Z = np.empty((Hs, S)); self.N = np.empty((Hs, S, dh))
        cm = np.empty((Hs, S))
        for a in range(Hs):
            self.m[a], self.Z[a], self.N[a], cm[a] = dense_causal_attention(
                self.q[1][:, a, :], Kh[:, a, :], Vh[:, a, :])
        self.colmass[1] = cm
        if self.fixed_mass:
            self.P = np.stack([dense_causal_probs(self.q[1][:, a, :], Kh[:, a, :]) for a in range(Hs)])
            self.Ofm = np.einsum('hij,jhd->hid', self.P, Vh.astype(np.float64))
        self._store_output(1, rows)
        self.loop = 1

    def run_loop(self, r):
        """Loop r >= 2: a1 gate, a2 projections, a3 residual quantisation,
        a4 column selection, a6 sparse update, a7 output projection."""
        assert r == self.loop + 1 and r >= 2
        S = self.S
        if self.token_budgets is None:
            rows = gate(self.X[r - 1], self.X[r - 2], self.active[r - 1], self.tau)
        else:
            rows = gate_topk(self.X[r - 1], self.X[r - 2], self.active[r - 1], self.token_budgets[r - 1])
        self.active[r] = rows
        k, v = self._project(r, rows)
        self.Kc.write_residual(r, rows, k)
        self.Vc.write_residual(r, rows, v)
        kr = self.kbud[r - 1]
        Hs = len(self.heads)
        T = []
        for a in range(Hs):
            if r == 2:
                cand = np.arange(S)
            else:
                cand = self.T[r - 1][a]
            if r > 2 and kr >= len(cand):
                T.append(np.asarray(cand, dtype=np.int64))
            else:
                T.append(topk_columns(self.colmass[r - 1][a].astype(np.float32), cand, kr))
        self.T[r] = T
        cm = np.zeros((Hs, S))
        for a in range(Hs):
            Ta = T[a]
            Ko = self.Kc.reconstruct(Ta, r - 1)[:, a, :]
            Kn = self.Kc.reconstruct(Ta, r)[:, a, :]
            Vo = self.Vc.reconstruct(Ta, r - 1)[:, a, :]
            Vn = self.Vc.reconstruct(Ta, r)[:, a, :]
            if self.fixed_mass:
                cm[a, Ta] = fixed_mass_update(rows, Ta, self.q[r][rows, a, :], Kn, Vo, Vn,
                                              self.P[a], self.Ofm[a])
                continue
            m2, Z2, N2, c = sparse_update(
                rows, Ta, self.q[r - 1][rows, a, :], self.q[r][rows, a, :],
                Ko, Kn, Vo, Vn, self.m[a, rows], self.Z[a, rows], self.N[a, rows])
            self.m[a, rows], self.Z[a, rows], self.N[a, rows] = m2, Z2, N2
            cm[a, Ta] = c
        self.colmass[r] = cm
        self._store_output(r, rows)
        self.loop = r

    def run(self, upto=None):
        upto = self.cfg.n_loops if upto is None else upto
        if self.loop == 0:
            self.run_loop1()
        while self.loop < upto:
            self.run_loop(self.loop + 1)
        return self


# --------------------------------------------------------------------------
# decode: one new token per sequence  [FL App. G: the decode selection is fused with the decode pass]
# --------------------------------------------------------------------------
class OracleDecode:
    """One decode token at position p = S_ctx against a context whose KV path
    (gate, projections, base and residual quantisation) ran for loops 1..R.

    The token is active at every loop.  Loop 1 attends densely over
    [0, p] on the reconstructed base; its own loop-1 probabilities, rounded
    to float32, select k columns per head (ties to the lower index).  Loops
    r >= 2 apply the sparse update over those columns.
    """

    def __init__(self, cfg, W, Xctx, xtok, heads=None, topk=None, quantize=True):
        self.cfg = cfg
        self.W = W
        self.p = cfg.seq
        self.dh = cfg.head_dim
        self.heads = list(range(cfg.n_heads)) if heads is None else list(heads)
        self.all_heads = len(self.heads) == cfg.n_heads
        self.k = cfg.k if topk is None else topk
        P1 = self.p + 1
        Hs = len(self.heads)
        self.Kc = KVStream(P1, Hs, self.dh, cfg.bits, quantize)
        self.Vc = KVStream(P1, Hs, self.dh, cfg.bits, quantize)
        self.Xctx, self.xtok = Xctx, xtok
        self.ctx_active = {}
        self.T = None
        self.O = {}
        self.Y = {}
        self.state = {}
        self.q = {}
        self.probs = None

    def prepare_context(self):
        """The context tokens' part of every loop (gate, k/v), which depends on
        the context alone: a decode reads it from the cache its prefill left."""
        self._ctx_kv = {r: self._context_kv(r) for r in range(1, self.cfg.n_loops + 1)}
        return self

    def _context_kv(self, r):
        """Context tokens' part of loop r: gate, k/v (no attention)."""
        if getattr(self, "_ctx_kv", None) and r in self._ctx_kv:
            return self._ctx_kv[r]
        cfg = self.cfg
        S = cfg.seq
        if r == 1:
            rows = np.arange(S)
        else:
            rows = gate(self.Xctx[r - 1], self.Xctx[r - 2], self.ctx_active[r - 1], cfg.tau)
        self.ctx_active[r] = rows
        _, k, v = project_qkv(self.Xctx[r - 1][rows], rows, self.W, self.heads, self.dh,
                              cfg.rope_theta)
        return rows, k, v

    def run(self):
        cfg, p, dh = self.cfg, self.p, self.dh
        Hs = len(self.heads)
        pos = np.array([p])
        q_prev = None
        for r in range(1, cfg.n_loops + 1):
            rows, kc, vc = self._context_kv(r)
            qt, kt, vt = project_qkv(self.xtok[r - 1][None, :], pos, self.W, self.heads, dh,
                                     cfg.rope_theta)
            all_rows = np.concatenate([rows, pos])
            kall = np.concatenate([kc, kt], axis=0)
            vall = np.concatenate([vc, vt], axis=0)
            if r == 1:
                self.Kc.write_base(kall)
                self.Vc.write_base(vall)
            else:
                self.Kc.write_residual(r, all_rows, kall)
                self.Vc.write_residual(r, all_rows, vall)
            if r == 1:
                cols = np.arange(p + 1)
                Kh = self.Kc.reconstruct(cols, 1)
                Vh = self.Vc.reconstruct(cols, 1)
                m = np.empty(Hs); Z = np.empty(Hs); N = np.empty((Hs, dh))
                probs = np.empty((Hs, p + 1))
                q = bf16_vals(qt)[0]
                for a in range(Hs):
                    s = (Kh[:, a, :].astype(np.float64) @ q[a]) / math.sqrt(dh)
                    m[a] = s.max()
                    e = np.exp(s - m[a])
                    Z[a] = e.sum()
                    N[a] = e @ Vh[:, a, :]
                    probs[a] = e / Z[a]
                self.probs = probs
                self.T = [topk_columns(probs[a].astype(np.float32), cols, self.k) for a in range(Hs)]
            else:
                for a in range(Hs):
                    Ta = self.T[a]
                    m2, Z2, N2, _ = sparse_update(
                        pos, Ta, q_prev[:, a, :], qt[:, a, :],
                        self.Kc.reconstruct(Ta, r - 1)[:, a, :], self.Kc.reconstruct(Ta, r)[:, a, :],
                        self.Vc.reconstruct(Ta, r - 1)[:, a, :], self.Vc.reconstruct(Ta, r)[:, a, :],
                        m[a:a + 1], Z[a:a + 1], N[a:a + 1])
                    m[a], Z[a], N[a] = m2[0], Z2[0], N2[0]
            q_prev = qt
            self.q[r] = qt[0]
            O = to_bf16_bits((N / Z[:, None]).reshape(1, Hs * dh))
            self.O[r] = O[0]
            self.state[r] = (m.copy(), Z.copy(), N.copy())
            if self.all_heads:
                self.Y[r] = out_projection(O, self.W["wo"])[0]
        return self


# --------------------------------------------------------------------------
# byte accounting  [FL §4.3, App. D.3; FZ §1 Cell 1 and §3 Cell 3]
# --------------------------------------------------------------------------
def cache_bytes(S, n_heads, head_dim, bits_per_loop, n_per_loop, group=GROUP, scale_bytes=2):
    """Bytes of the K and V caches: the loop-1 base over all S tokens and the
    loop-l residual streams over their n_l active tokens (codes plus one
    scale per group).  Returns (base, [loop 2, loop 3, ...])."""
    def per_token(bits):
        return 2 * n_heads * (head_dim * bits // 8 + scale_bytes * (head_dim // group))
    base = S * per_token(bits_per_loop[0])
    loops = [n_per_loop[l] * per_token(bits_per_loop[l]) for l in range(1, len(bits_per_loop))]
    return base, loops


def dense_kv_bytes(S, n_heads, head_dim, n_loops, layers=1, elem_bytes=2):
    """Bytes of an uncompressed per-loop KV cache (K and V, every loop)."""
    return 2 * n_loops * S * n_heads * head_dim * elem_bytes * layers


def first_order_storage(S, elems_per_token_loop, base_bits, residual_bits, residual_fracs,
                        tail_tokens, tail_bytes=2):
    """First-order storage of a base-plus-residual cache with no quantisation
    metadata: a base over all S tokens, one residual per loop over the
    active fraction of tokens, and a recent-token tail kept in 16-bit.
    Returns (base, residuals, tail) in bytes."""
    base = S * elems_per_token_loop * base_bits / 8
    res = sum(S * f * elems_per_token_loop * residual_bits / 8 for f in residual_fracs)
    tail = tail_tokens * elems_per_token_loop * tail_bytes
    return base, res, tail
