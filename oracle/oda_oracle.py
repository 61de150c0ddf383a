"""Oracle for the On-Demand Attention (ODA) decode path and the Declarative Attention (DA)
block-mask path: a plain, slow, fp64 CPU restatement of what the path computes.

TEST INFRASTRUCTURE ONLY. Only the tests, the package's smoke check and the bench's CPU
baseline leg may import this module. The product path never calls it, and it shares no
code with the CUDA library (it reads inputs from the seeded generator module only).

Sources (page titles; sections as printed on each page):
  [ODA]  "On-Demand Attention: Language Models Know When to Recall" (arxiv-wiki summary),
         sections 접근 방법 (approach), 주요 결과 (results), 개발자 관점 (developer view).
  [DA]   "[논문리뷰] Language Models Can Control Their Own Attention", section 3
         (method & key results), and its abstract page ("언어 모델은 자신의 어텐션을 제어할
         수 있다").

Readings where the pages are silent (each is listed in the design notes):
  * Attention is plain scaled-dot-product softmax attention, scale 1/sqrt(d), natural-log
    normaliser; query head h reads KV head floor(h / G) (grouped-query attention).
  * Local = the first s positions plus the w most recent positions, the current one
    included, as a set union (no position counted twice).
  * The recall head is a 2-layer MLP, x = [h_{t-1}; E(x_t); h^L_t], z = W1^T x + b1,
    a = GELU(z) with the exact erf form, q = w2 . a + b2; evaluated here in fp64.
  * Gate: Full is recomputed iff q > theta (strict), theta = 0 by default.
  * DA blocks: a requested token region keeps every 16-token page it touches; positions
    after the current one are never visible.

Every function below is pinned by tests/test_oracle_pins.py against closed forms,
invariants, library routines or brute force; the one exception is marked
"parity unpinned" (none at present).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 16          # paged-KV page size in tokens
DEFAULT_SINK = 4    # [ODA] 접근 방법: initial s = 4 tokens
DEFAULT_WINDOW = 2048  # [ODA] 접근 방법 / 주요 결과: recent w = 2048, current token included
DEFAULT_THETA = 0.0    # [ODA] 접근 방법: q_t > theta, theta = 0 by default


# ----------------------------------------------------------------------------------------
# Inputs: bf16 bit patterns widened exactly to fp64.
# ----------------------------------------------------------------------------------------
def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):          # NaN payloads widen to NaN
        return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------------------
# Visible position sets.
# ----------------------------------------------------------------------------------------
def full_positions(t: int) -> np.ndarray:
    """Full attention at position t sees the whole retained history 0..t ([ODA] 접근 방법:
    Full over the complete history)."""
    return np.arange(t + 1, dtype=np.int64)


def local_positions(t: int, sink: int = DEFAULT_SINK, window: int = DEFAULT_WINDOW) -> np.ndarray:
    """Local attention at position t: the first `sink` positions and the `window` most
    recent positions, the current position counted inside the window ([ODA] 접근 방법 and
    주요 결과). Overlap is a plain set union."""
    sink_end = min(sink, t + 1)
    win_start = max(0, t - window + 1)
    if win_start <= sink_end:
        return np.arange(t + 1, dtype=np.int64)
    return np.concatenate([np.arange(sink_end, dtype=np.int64),
                           np.arange(win_start, t + 1, dtype=np.int64)])


def check_keep_list(t: int, keep_blocks, block: int = BLOCK) -> None:
    """A keep list names logical pages, strictly ascending, each at or before page t//block."""
    k = np.asarray(keep_blocks, dtype=np.int64)
    if k.size and (k[0] < 0 or k[-1] > t // block or np.any(np.diff(k) <= 0)):
        raise ValueError("keep list must be strictly ascending logical pages within 0..t//16")


def keep_positions(t: int, keep_blocks, block: int = BLOCK) -> np.ndarray:
    """[DA] section 3: the engine rewrites the block table so that only kept pages reach the
    attention kernel. Visible = every position of a kept page, up to the current one."""
    check_keep_list(t, keep_blocks, block)
    parts = [np.arange(b * block, min(b * block + block, t + 1), dtype=np.int64)
             for b in np.asarray(keep_blocks, dtype=np.int64)]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def da_mode_positions(mode: int, t: int, focus_offset: int = 0, *, focus_len: int = 32768,
                      recent: int = 2048, local_len: int = 4096, block: int = BLOCK) -> np.ndarray:
    """[DA] three declared modes, as token regions rounded out to whole pages:
    global (0) = the whole context; focus (1) = the sink page, one focused region
    [off, off + focus_len) and the `recent` latest tokens; local (2) = the `local_len`
    latest tokens only. A region keeps every page it touches; nothing after t is visible."""
    if mode == 0:
        regions = [(0, t)]
    elif mode == 1:
        if focus_offset < 0:
            raise ValueError("the focused region starts at a position, >= 0")
        regions = [(0, 0), (focus_offset, min(t, focus_offset + focus_len - 1)),
                   (max(0, t - recent + 1), t)]
    elif mode == 2:
        regions = [(max(0, t - local_len + 1), t)]
    else:
        raise ValueError("mode must be 0 (global), 1 (focus) or 2 (local)")
    visible = np.zeros(t + 1, dtype=bool)
    for lo, hi in regions:
        if lo > hi:
            continue
        first = (lo // block) * block
        last = min(t, (hi // block) * block + block - 1)
        visible[first:last + 1] = True
    return np.nonzero(visible)[0].astype(np.int64)


def shard_positions(t: int, lo: int, hi: int) -> np.ndarray:
    """One GPU's part of a context-parallel Full: the positions of 0..t inside [lo, hi)."""
    return np.arange(max(lo, 0), min(hi, t + 1), dtype=np.int64)


# ----------------------------------------------------------------------------------------
# Paged KV reads.
# ----------------------------------------------------------------------------------------
def paged_rows(cache_bits, block_row, positions, kv_head: int, block: int = BLOCK) -> np.ndarray:
    """Rows of one KV head at logical positions, read through one sequence's block table.
    cache_bits: uint16 [num_pages][Hkv][block][d]; block_row: physical page per logical page."""
    p = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(block_row, dtype=np.int64)[p // block]
    return widen_bf16(cache_bits[pages, kv_head, p % block, :])


# ----------------------------------------------------------------------------------------
# Attention.
# ----------------------------------------------------------------------------------------
def softmax_attention(q, K, V, scale: float):
    """o = sum_p w_p v_p with w = softmax(scale * K q), and the natural-log normaliser
    lse = log sum_p exp(scale * k_p . q). An empty set gives o = 0, lse = -inf."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1] if V.ndim == 2 else q.shape[0]), -math.inf
    s = (K @ q) * scale
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    return (e @ V) / z, m + math.log(z)


def decode_attention(q_heads, k_rows, v_rows, scale: float):
    """One sequence, one layer. q_heads: fp64 [Hq][d]; k_rows / v_rows: fp64
    [Hkv][n][d] over the visible positions. Query head h reads KV head h // (Hq / Hkv).
    Returns out [Hq][d] and lse [Hq]."""
    q_heads = np.asarray(q_heads, dtype=np.float64)
    Hq, d = q_heads.shape
    Hkv = len(k_rows)
    G = Hq // Hkv
    out = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for h in range(Hq):
        out[h], lse[h] = softmax_attention(q_heads[h], k_rows[h // G], v_rows[h // G], scale)
    return out, lse


# ----------------------------------------------------------------------------------------
# Recall head and gate.
# ----------------------------------------------------------------------------------------
def lse_merge(parts):
    """Combine attention results over disjoint position sets: parts = [(o_r, lse_r)], each o_r
    normalised over its own set, lse_r its natural-log normaliser (-inf: empty set). The
    union's result is sum_r e^(lse_r - M) o_r / sum_r e^(lse_r - M), M = max lse_r, with
    normaliser M + log sum_r e^(lse_r - M); all parts empty gives (0, -inf)."""
    lses = [float(l) for _, l in parts]
    m = max(lses)
    if m == -math.inf:
        return np.zeros_like(np.asarray(parts[0][0], dtype=np.float64)), -math.inf
    w = [0.0 if l == -math.inf else math.exp(l - m) for l in lses]
    total = sum(w)
    o = sum(wr * np.asarray(o_r, dtype=np.float64) for wr, (o_r, _) in zip(w, parts)) / total
    return o, m + math.log(total)


def gelu(z):
    """Exact GELU: z * Phi(z) = z/2 (1 + erf(z / sqrt 2))."""
    z = np.asarray(z, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def recall_score(h_prev, emb, h_local, W1, b1, w2, b2):
    """[ODA] 접근 방법: the recall head reads the previous selected hidden state h_{t-1},
    the current token's embedding E(x_t) and the current Local final hidden h^L_t, and
    returns a scalar q_t. Batched over rows; inputs [B][D], W1 [3D][M], b1 [M], w2 [M]."""
    x = np.concatenate([np.asarray(h_prev, np.float64), np.asarray(emb, np.float64),
                        np.asarray(h_local, np.float64)], axis=-1)
    z = x @ np.asarray(W1, np.float64) + np.asarray(b1, np.float64)
    return gelu(z) @ np.asarray(w2, np.float64) + float(b2)


def random_schedule_gate(u, rho: float):
    """[ODA] 주요 결과, the random-timing ablation: Full is called with probability rho at
    each (sequence, step), independently of the state; u are the caller's uniform draws."""
    return np.asarray(u, dtype=np.float64) < rho


def gate(q, theta: float = DEFAULT_THETA):
    """[ODA] 접근 방법: recompute with Full iff q_t > theta (strict)."""
    return np.asarray(q, dtype=np.float64) > theta


# ----------------------------------------------------------------------------------------
# Recall-head training objective ([ODA] 핵심 기여 and 접근 방법: the gain of Full over Local
# g_t = log p^F - log p^L, its cost-adjusted form d_t = g_t - lambda, the signed-log target
# y_t = sign(d_t) log(1 + |d_t|), and Huber regression with delta = 1 of q_t on y_t).
# ----------------------------------------------------------------------------------------
def signed_log_target(gain, lam: float):
    """y = sign(d) log(1 + |d|) with d = gain - lambda."""
    d = np.asarray(gain, dtype=np.float64) - lam
    return np.sign(d) * np.log1p(np.abs(d))


def huber(r, delta: float = 1.0):
    """r^2 / 2 for |r| <= delta, delta (|r| - delta / 2) beyond."""
    r = np.asarray(r, dtype=np.float64)
    a = np.abs(r)
    return np.where(a <= delta, 0.5 * r * r, delta * (a - 0.5 * delta))


def gelu_grad(z):
    """d/dz of z Phi(z): Phi(z) + z phi(z)."""
    z = np.asarray(z, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * (1.0 + erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)


def recall_loss_grad(h_prev, emb, h_local, W1, b1, w2, b2, gain, lam: float, delta: float = 1.0):
    """Mean Huber loss of the recall head over a batch and its gradient with respect to the
    head's parameters (the backbone is frozen). The pages do not print the reduction; the
    batch mean is taken. Returns (loss, q [B], dW1 [3D][M], db1 [M], dw2 [M], db2)."""
    x = np.concatenate([np.asarray(h_prev, np.float64), np.asarray(emb, np.float64),
                        np.asarray(h_local, np.float64)], axis=-1)
    W1, b1, w2 = (np.asarray(a, np.float64) for a in (W1, b1, w2))
    z = x @ W1 + b1
    a = gelu(z)
    q = a @ w2 + float(b2)
    y = signed_log_target(gain, lam)
    r = q - y
    B = x.shape[0]
    loss = float(huber(r, delta).sum() / B)
    dq = np.clip(r, -delta, delta) / B            # d loss / d q_b
    dw2 = a.T @ dq
    db2 = float(dq.sum())
    dz = np.outer(dq, w2) * gelu_grad(z)          # [B][M]
    db1 = dz.sum(axis=0)
    dW1 = x.T @ dz
    return loss, q, dW1, db1, dw2, db2


# ----------------------------------------------------------------------------------------
# Cost model.
# ----------------------------------------------------------------------------------------
def attended_tokens(t: int, gated: bool, sink: int = DEFAULT_SINK,
                    window: int = DEFAULT_WINDOW) -> int:
    """Tokens attended per head at position t: the Local set always, plus the whole
    history when the step is recomputed with Full ([ODA] 접근 방법: Local first, Full on
    demand)."""
    return len(local_positions(t, sink, window)) + (t + 1 if gated else 0)


def attention_cost_ratio(n: int, out_len: int, rho: float, sink: int = DEFAULT_SINK,
                         window: int = DEFAULT_WINDOW) -> float:
    """[ODA] 접근 방법, last item: Local costs a fixed ell = s + w, Full grows linearly with
    the history n, and the average cost follows from the Full-call rate rho. Exact
    attention-only ratio ODA / Full over a generation of out_len tokens after n:
    sum_t (min(t+1, ell) + rho (t+1)) / sum_t (t+1), t = n .. n+out_len-1."""
    ell = sink + window
    ts = np.arange(n, n + out_len, dtype=np.float64)
    return float((np.minimum(ts + 1, ell).sum() + rho * (ts + 1).sum()) / (ts + 1).sum())


# ----------------------------------------------------------------------------------------
# One ODA decode step over an attention-only stack.
# ----------------------------------------------------------------------------------------
class OdaDecoder:
    """The ODA step ([ODA] 접근 방법 and 개발자 관점), over an attention-only stack whose
    per-layer Q/K/V are given as inputs:
      1. Local at every layer, over the prior cache plus the Local K/V at slot t (a layer
         outside the Local restriction -- hybrid backbones restrict only some layers, [ODA]
         개발자 관점 -- attends all of 0..t here too; s and w may differ per layer);
      2. q_t from the recall head on (h_{t-1}, E(x_t), last layer's Local output);
      3. where q_t > theta, Full at every layer over the same prior cache plus the Full
         K/V at slot t, replacing the Local result;
      4. the selected path's K/V is committed at slot t; h_{t-1} <- selected last output.
    The cache is kept in logical position order, bf16 bits: k[l][b][g][p][:]."""

    def __init__(self, k_hist_bits, v_hist_bits, lengths, h_prev, recall, *,
                 sink=DEFAULT_SINK, window=DEFAULT_WINDOW, theta=DEFAULT_THETA, scale=None,
                 local_layers=None, sinks=None, windows=None, random_rho=None):
        self.k = [np.array(x, dtype=np.uint16) for x in k_hist_bits]   # per layer [B][Hkv][cap][d]
        self.v = [np.array(x, dtype=np.uint16) for x in v_hist_bits]
        self.lengths = list(lengths)
        self.h_prev = np.asarray(h_prev, dtype=np.float64)
        self.W1, self.b1, self.w2, self.b2 = recall
        self.sink, self.window, self.theta = sink, window, theta
        L = len(self.k)
        self.local_layers = [True] * L if local_layers is None else [bool(x) for x in local_layers]
        self.sinks = [sink] * L if sinks is None else list(sinks)
        self.windows = [window] * L if windows is None else list(windows)
        self.random_rho = random_rho     # not None: the random-timing ablation decides
        d = self.k[0].shape[-1]
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale

    def _attend(self, layer, b, t, positions, q_bits, k_new_bits, v_new_bits):
        Hkv = self.k[layer].shape[1]
        hist = positions[positions < t]
        ks, vs = [], []
        for g in range(Hkv):
            kr = widen_bf16(self.k[layer][b, g, hist])
            vr = widen_bf16(self.v[layer][b, g, hist])
            if positions.size and positions[-1] == t:
                kr = np.vstack([kr, widen_bf16(k_new_bits[g])[None]])
                vr = np.vstack([vr, widen_bf16(v_new_bits[g])[None]])
            ks.append(kr)
            vs.append(vr)
        return decode_attention(widen_bf16(q_bits), ks, vs, self.scale)

    def step(self, inp, gate_hint=None, near=1e-3):
        """inp: dict of bf16-bit arrays q_local/k_local/v_local/q_full/k_full/v_full, each a
        list over layers of [B][H][d], emb fp64 [B][D] and, for the random schedule, gate_u
        [B]. gate_hint: the device's gate, used
        only where |q - theta| < near so that a rounding-level tie cannot fork the history.
        Returns (out [L][B][Hq][d], lse [L][B][Hq], q [B], gate [B])."""
        L = len(self.k)
        B = len(self.lengths)
        Hq = inp["q_local"][0].shape[1]
        d = self.k[0].shape[-1]
        out = np.zeros((L, B, Hq, d))
        lse = np.zeros((L, B, Hq))
        for layer in range(L):
            for b in range(B):
                t = self.lengths[b]
                if self.local_layers[layer]:
                    pos = local_positions(t, self.sinks[layer], self.windows[layer])
                else:
                    pos = full_positions(t)
                out[layer, b], lse[layer, b] = self._attend(
                    layer, b, t, pos, inp["q_local"][layer][b],
                    inp["k_local"][layer][b], inp["v_local"][layer][b])
        h_local = out[L - 1].reshape(B, Hq * d)
        q = recall_score(self.h_prev, inp["emb"], h_local, self.W1, self.b1, self.w2, self.b2)
        g = gate(q, self.theta)
        if self.random_rho is not None:
            g = random_schedule_gate(inp["gate_u"], self.random_rho)
        elif gate_hint is not None:
            hint = np.asarray(gate_hint, dtype=bool)
            tie = np.abs(q - self.theta) < near
            g = np.where(tie, hint, g)
        for b in range(B):
            if not g[b]:
                continue
            t = self.lengths[b]
            pos = full_positions(t)
            for layer in range(L):
                out[layer, b], lse[layer, b] = self._attend(
                    layer, b, t, pos, inp["q_full"][layer][b],
                    inp["k_full"][layer][b], inp["v_full"][layer][b])
        for layer in range(L):
            for b in range(B):
                t = self.lengths[b]
                src = "full" if g[b] else "local"
                self.k[layer][b, :, t] = inp["k_" + src][layer][b]
                self.v[layer][b, :, t] = inp["v_" + src][layer][b]
        self.lengths = [x + 1 for x in self.lengths]
        self.h_prev = out[L - 1].reshape(B, Hq * d).copy()
        return out, lse, q, g
