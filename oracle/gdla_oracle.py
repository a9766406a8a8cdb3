"""GDLA forward oracle: a plain, slow, float64 CPU statement of the layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this
module; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg
of ``bench.py`` use it.  It shares no code with the CUDA path (it does not import the
``differential_latent_attention_fwd_b200`` package; callers hand it plain arrays).

Source of every step: "Motif 3: Technical Report", picx.dev summary page, section 2.2
"Grouped Differential Latent Attention (GDLA)" (equations for c^Q, [q^C; q^R], [c^KV; k^R],
the normalised latent, [K^C; V], the head split n_N = n_H/(g+1), lambda_t, D_t, G_t and the
gated output), plus the paperglide.net page ("Model Architecture" worked example and the
Figure 1 caption: one lambda per signal head, gate from the normalised query latent, one
rotary key shared by all KV heads, 16 KV heads shared by the signal and noise paths).

Every floating-point step is float64.  Matrix products use numpy's BLAS or torch's CPU
matmul (library primitives); the masked softmax uses torch.softmax (a library routine).  The only grouping beyond the equations: prefill evaluates the masked softmax
attention of several query rows as one product over a shared key block (each row still
normalises over exactly its own visible keys), and the weight-absorbed decode route is a
second, independent statement of the same algebra, checked against the literal one.

Readings where the pages are silent (each also listed in the design notes):
  * weights are [in, out] (the pages write x W);
  * [q^C; q^R]: the first n_H*d_nope columns are q^C (head-major), the rest q^R (head-major);
  * [c^KV; k^R]: the first kv_rank columns are c^KV, the last d_rope are k^R;
  * Reshape_heads(c W_b^KV): head j owns columns j*(d_nope+d_v) ..., K^C first then V;
  * heads 0..n_S-1 are the signal heads, n_S..n_H-1 the noise heads; signal head s reads
    KV head s // (n_S/n_KV), noise head n reads KV head n // (n_N/n_KV);
  * Repeat_g pairs signal head s with noise head s // g ("grouped"); the paperglide worked
    example lists the noise outputs tiled (s mod n_N), available as noise_map="tiled";
  * softmax scale 1/sqrt(d_nope + d_rope); RMSNorm eps 1e-6 with a gain vector;
  * RoPE: rotate-half on the d_rope part, pairs (i, i + d_rope/2), angle pos * theta^(-2i/d_rope),
    theta 10000, pos = 0-based token index (decode: the number of cached keys);
  * masks: causal s <= t; sliding window t - W < s <= t (W keys, self included);
  * no biases, no per-head normalisation after the subtraction; vec() is head-major.

Parity: every function here is pinned by tests/test_oracle_pins.py (worked example, closed
forms, library routines, invariants, brute force) except where a docstring says otherwise.
Parity unpinned by the pages: the constants taken where the pages are silent (the softmax
scale 1/sqrt(192), the rotate-half RoPE pairing with theta 10000, the RMSNorm eps) are
readings, not printed values; the pins fix the forms these steps take (a rotation, a norm, a
softmax), and the kernels share the constants by construction, not by a check against the
pages.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


# --------------------------------------------------------------------------------------
# configuration
# --------------------------------------------------------------------------------------
@dataclass(frozen=True)
class OracleConfig:
    d_model: int
    q_rank: int
    kv_rank: int
    n_signal: int
    n_noise: int
    n_kv_heads: int
    d_nope: int
    d_rope: int
    d_v: int
    window: int = 0
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    noise_map: str = "grouped"      # Repeat_g order: "grouped" (s // g) or "tiled" (s % n_N)

    @property
    def n_heads(self) -> int:
        return self.n_signal + self.n_noise

    @property
    def g(self) -> int:
        """Grouped ratio: n_N = n_H / (g + 1), n_S = g n_N (picx.dev page, section 2.2)."""
        assert self.n_heads % (self.n_noise) == 0
        g = self.n_heads // self.n_noise - 1
        assert self.n_signal == g * self.n_noise
        return g

    @staticmethod
    def from_shape(s, noise_map: str = "grouped") -> "OracleConfig":
        """Build from any object with the same attribute names (e.g. synth.GdlaShape)."""
        return OracleConfig(s.d_model, s.q_rank, s.kv_rank, s.n_signal, s.n_noise, s.n_kv_heads,
                            s.d_nope, s.d_rope, s.d_v, s.window, s.rope_theta, s.rms_eps,
                            noise_map)


def f64(a) -> np.ndarray:
    """Exact upcast of a torch tensor (any dtype, incl. bf16) or array-like to float64."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # local: the oracle needs torch only to read tensors it is handed
        return a.to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------------------
# element-wise building blocks
# --------------------------------------------------------------------------------------
def rms_norm(v: np.ndarray, gain: np.ndarray | None, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: v / sqrt(mean(v^2) + eps) * gain."""
    r = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return r if gain is None else r * gain


def rope(v: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding of the decoupled rope part (last axis, even length).

    Pair (i, i + d/2) is rotated by angle pos * theta^(-2i/d).  ``pos`` broadcasts against
    ``v[..., 0]``.
    """
    d = v.shape[-1]
    half = d // 2
    inv_freq = theta ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = v[..., :half], v[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function, evaluated without overflow for either sign."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


# --------------------------------------------------------------------------------------
# head bookkeeping
# --------------------------------------------------------------------------------------
def kv_head_of(cfg: OracleConfig) -> np.ndarray:
    """KV head read by each of the n_H query heads (signal heads first, then noise heads)."""
    assert cfg.n_signal % cfg.n_kv_heads == 0 and cfg.n_noise % cfg.n_kv_heads == 0
    sig = np.arange(cfg.n_signal) // (cfg.n_signal // cfg.n_kv_heads)
    noi = np.arange(cfg.n_noise) // (cfg.n_noise // cfg.n_kv_heads)
    return np.concatenate([sig, noi])


def noise_of_signal(cfg: OracleConfig) -> np.ndarray:
    """Repeat_g: the noise head whose output signal head s subtracts."""
    s = np.arange(cfg.n_signal)
    if cfg.noise_map == "grouped":
        return s // cfg.g
    if cfg.noise_map == "tiled":
        return s % cfg.n_noise
    raise ValueError(cfg.noise_map)


def key_range(t: int, window: int) -> tuple[int, int]:
    """Keys visible to query position t: [lo, t] (causal, or the last ``window`` keys)."""
    lo = 0 if window <= 0 else max(0, t - window + 1)
    return lo, t


# --------------------------------------------------------------------------------------
# projections (picx.dev page, section 2.2, first five equations)
# --------------------------------------------------------------------------------------
def query_path(x: np.ndarray, W_aQ, W_bQ, g_q, pos, cfg: OracleConfig):
    """c^Q = RMSNorm(x W_aQ); [q^C; q^R] = c^Q W_bQ; RoPE on q^R.

    x: [N, d].  Returns (c^Q [N, r_q], q^C [N, n_H, d_nope], rotated q^R [N, n_H, d_rope]).
    """
    cQ = rms_norm(x @ W_aQ, g_q, cfg.rms_eps)
    qq = cQ @ W_bQ
    nc = cfg.n_heads * cfg.d_nope
    qC = qq[:, :nc].reshape(-1, cfg.n_heads, cfg.d_nope)
    qR = qq[:, nc:].reshape(-1, cfg.n_heads, cfg.d_rope)
    qR = rope(qR, np.asarray(pos)[:, None], cfg.rope_theta)
    return cQ, qC, qR


def kv_latent(x: np.ndarray, W_aKV, g_kv, pos, cfg: OracleConfig):
    """[c^KV; k^R] = x W_aKV; normalised latent = RMSNorm(c^KV); RoPE on k^R (not normalised).

    Returns (c_bar [N, kv_rank], rotated k^R [N, d_rope]); together they are one latent-cache row.
    """
    ck = x @ W_aKV
    cbar = rms_norm(ck[:, : cfg.kv_rank], g_kv, cfg.rms_eps)
    kR = rope(ck[:, cfg.kv_rank:], np.asarray(pos), cfg.rope_theta)
    return cbar, kR


def kv_heads(cbar: np.ndarray, W_bKV, cfg: OracleConfig):
    """[K^C; V] = Reshape_heads(c_bar W_bKV) -> K^C [N, n_KV, d_nope], V [N, n_KV, d_v]."""
    kv = (cbar @ W_bKV).reshape(-1, cfg.n_kv_heads, cfg.d_nope + cfg.d_v)
    return kv[..., : cfg.d_nope], kv[..., cfg.d_nope:]


def lambda_coeff(x: np.ndarray, W_lambda) -> np.ndarray:
    """lambda_t = sigmoid(x_t W^lambda), one value per signal head."""
    return sigmoid(x @ W_lambda)


def gate_logits(cQ: np.ndarray, W_G, cfg: OracleConfig) -> np.ndarray:
    """G_t = Reshape_heads(c^Q_t W^G) -> [N, n_S, d_v] (the sigmoid is applied in the combine)."""
    return (cQ @ W_G).reshape(-1, cfg.n_signal, cfg.d_v)


# --------------------------------------------------------------------------------------
# attention, combine, output
# --------------------------------------------------------------------------------------
def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Textbook softmax attention of a few queries over one key set.

    q [h, dk], k [S, dk], v [S, dv] -> [h, dv] = softmax(q k^T * scale) v.
    """
    s = (q @ k.T) * scale
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ v


def differential_combine(H_S: np.ndarray, H_N: np.ndarray, lam: np.ndarray,
                         gate: np.ndarray, noise_map: np.ndarray, gate_is_logit: bool = True):
    """D = H_S - lambda (.) Repeat_g(H_N); returns (D, sigmoid(G) (.) D).

    H_S [n_S, dv], H_N [n_N, dv], lam [n_S], gate [n_S, dv] (logits G, or already-sigmoided
    values when ``gate_is_logit`` is False), noise_map [n_S] = noise head of each signal head.
    """
    D = H_S - lam[:, None] * H_N[noise_map]
    sg = sigmoid(gate) if gate_is_logit else gate
    return D, sg * D


def attend_row(qC_t, qR_t, KC, kR, V, lo: int, hi: int, cfg: OracleConfig) -> np.ndarray:
    """Per-head attention outputs H [n_H, d_v] of one query over keys lo..hi (inclusive).

    q_h = [q^C_h; q^R_h], k_{j,s} = [K^C_{j,s}; k^R_s] (one rotary key for all KV heads).
    """
    scale = 1.0 / np.sqrt(cfg.d_nope + cfg.d_rope)
    kvh = kv_head_of(cfg)
    H = np.empty((cfg.n_heads, cfg.d_v))
    kR_keys = kR[lo: hi + 1]
    for j in range(cfg.n_kv_heads):
        heads = np.nonzero(kvh == j)[0]
        q = np.concatenate([qC_t[heads], qR_t[heads]], axis=-1)
        k = np.concatenate([KC[lo: hi + 1, j], kR_keys], axis=-1)
        H[heads] = softmax_attention(q, k, V[lo: hi + 1, j], scale)
    return H


def combine_row(H: np.ndarray, lam_t: np.ndarray, G_t: np.ndarray, W_O, cfg: OracleConfig):
    """Differential combine + sigmoid gate + output projection of one token: returns (Dg, y)."""
    _, Dg = differential_combine(H[: cfg.n_signal], H[cfg.n_signal:], lam_t, G_t,
                                 noise_of_signal(cfg))
    return Dg, Dg.reshape(-1) @ W_O


# --------------------------------------------------------------------------------------
# full layer: prefill
# --------------------------------------------------------------------------------------
def _weights64(w: dict) -> dict:
    return {k: f64(v) for k, v in w.items()}


def masked_softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                             allowed: np.ndarray) -> np.ndarray:
    """Masked softmax attention of several query rows over one shared key block.

    q [r, h, dk] (r query positions, h heads reading the same keys), k [S, dk], v [S, dv],
    allowed [r, S] bool (key s visible to row r) -> [r, h, dv] = softmax(q k^T scale + mask) v.
    Every row must see at least one key.  Evaluated with float64 torch CPU ops (matmul,
    masked fill, softmax), which run multithreaded on large blocks.
    """
    import torch
    r, h, dk = q.shape
    tq, tk, tv = torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)
    s = (tq.reshape(r * h, dk) @ tk.T).reshape(r, h, -1) * scale
    s.masked_fill_(~torch.from_numpy(allowed)[:, None, :], float("-inf"))
    p = torch.softmax(s, dim=-1)
    return (p.reshape(r * h, -1) @ tv).reshape(r, h, -1).numpy()


def _row_chunks(rows, window: int, max_rows: int = 64):
    """Split sorted query rows into runs whose shared key span stays near what each row needs."""
    out, i = [], 0
    while i < len(rows):
        lo0 = key_range(rows[i], window)[0]
        k = i + 1
        while k < len(rows) and k - i < max_rows:
            t = rows[k]
            need = t - key_range(t, window)[0] + 1
            if t - lo0 + 1 > 2 * need + 1024:
                break
            k += 1
        out.append((i, k))
        i = k
    return out


def gdla_prefill(x, weights: dict, cfg: OracleConfig, rows=None, g_q=None, g_kv=None,
                 pos_offset: int = 0, return_parts: bool = False, chunk: int = 8192):
    """GDLA(x_t) for every sequence of a batch, at the requested query rows.

    x [B, T, d]; ``rows`` = list of query positions (default: all).  Position of token t is
    pos_offset + t.  Returns y [B, len(rows), d] (and a dict of per-row intermediates when
    ``return_parts``: c^Q, q^C, q^R, lambda, G, Dg and, for all tokens, c_bar, k^R, K^C, V).
    Attention is evaluated one KV head at a time for all requested rows (signal and noise
    heads of that KV head together), rows batched into masked products over a shared key
    block; each row's softmax still runs over exactly its own visible keys.
    """
    W = _weights64(weights)
    gq = None if g_q is None else f64(g_q)
    gkv = None if g_kv is None else f64(g_kv)
    B, T, _ = x.shape
    rows = list(range(T)) if rows is None else [int(r) for r in rows]
    rows_a = np.asarray(rows)
    order = np.argsort(rows_a, kind="stable")
    srows = rows_a[order]
    t_hi = int(srows[-1]) + 1
    scale = 1.0 / np.sqrt(cfg.d_nope + cfg.d_rope)
    kvh = kv_head_of(cfg)
    blk = cfg.d_nope + cfg.d_v
    chunks = _row_chunks(srows.tolist(), cfg.window)
    ys, parts = [], []
    for b in range(B):
        # latent rows (c_bar, k^R) of every token a requested query can see
        cbar = np.empty((t_hi, cfg.kv_rank))
        kR = np.empty((t_hi, cfg.d_rope))
        for c0 in range(0, t_hi, chunk):
            c1 = min(t_hi, c0 + chunk)
            xb = f64(x[b, c0:c1])
            cbar[c0:c1], kR[c0:c1] = kv_latent(xb, W["W_aKV"], gkv,
                                               pos_offset + np.arange(c0, c1), cfg)
        xr = f64(x[b, rows])
        pos_r = pos_offset + rows_a
        cQ, qC, qR = query_path(xr, W["W_aQ"], W["W_bQ"], gq, pos_r, cfg)
        lam = lambda_coeff(xr, W["W_lambda"])
        G = gate_logits(cQ, W["W_G"], cfg)
        H = np.empty((len(rows), cfg.n_heads, cfg.d_v))
        if return_parts:
            KC_all = np.empty((t_hi, cfg.n_kv_heads, cfg.d_nope))
            V_all = np.empty((t_hi, cfg.n_kv_heads, cfg.d_v))
        for j in range(cfg.n_kv_heads):
            heads = np.nonzero(kvh == j)[0]
            # [K^C_j; V_j] = c_bar W_b^KV restricted to KV head j's column block
            KC_j = cbar @ W["W_bKV"][:, j * blk: j * blk + cfg.d_nope]
            V_j = cbar @ W["W_bKV"][:, j * blk + cfg.d_nope: (j + 1) * blk]
            if return_parts:
                KC_all[:, j], V_all[:, j] = KC_j, V_j
            K_j = np.concatenate([KC_j, kR], axis=-1)           # k_{j,s} = [K^C_{j,s}; k^R_s]
            q_j = np.concatenate([qC[:, heads], qR[:, heads]], axis=-1)
            for i0, i1 in chunks:
                rr = srows[i0:i1]
                idx = order[i0:i1]
                los = np.array([key_range(int(t), cfg.window)[0] for t in rr])
                lo, hi = int(los.min()), int(rr.max())
                keys = np.arange(lo, hi + 1)
                allowed = (keys[None, :] >= los[:, None]) & (keys[None, :] <= rr[:, None])
                H[idx[:, None], heads[None, :]] = masked_softmax_attention(
                    q_j[idx], K_j[lo: hi + 1], V_j[lo: hi + 1], scale, allowed)
        y = np.empty((len(rows), cfg.d_model))
        Dg_all = np.empty((len(rows), cfg.n_signal, cfg.d_v))
        for i in range(len(rows)):
            Dg_all[i], y[i] = combine_row(H[i], lam[i], G[i], W["W_O"], cfg)
        ys.append(y)
        if return_parts:
            parts.append(dict(cQ=cQ, qC=qC, qR=qR, lam=lam, G=G, Dg=Dg_all,
                              cbar=cbar, kR=kR, KC=KC_all, V=V_all))
    y = np.stack(ys)
    return (y, parts) if return_parts else y


def gdla_prefill_after_prefix(x_local, prefix_latent, pos_offset: int, weights: dict,
                              cfg: OracleConfig, g_q=None, g_kv=None):
    """GDLA rows of the tokens x_local [T, d] at positions pos_offset .. pos_offset + T - 1 of
    one sequence whose n_prefix preceding tokens (positions pos_offset - n_prefix ..
    pos_offset - 1) are given only by their latent rows prefix_latent [n_prefix, kv_rank + d_rope]
    (c_bar | rotated k^R, as a cache row).  The definition of section 2.2 of the picx.dev page
    with the keys and values of those tokens expanded from the given rows; this is the unit a
    context-parallel rank computes (paperglide.net summary, Figure 5 caption: ranks exchange
    key/value information only).  Row by row, for small cases.  Returns y [T, d].
    """
    W = _weights64(weights)
    gq = None if g_q is None else f64(g_q)
    gkv = None if g_kv is None else f64(g_kv)
    x = f64(x_local)
    T = x.shape[0]
    pre = np.zeros((0, cfg.kv_rank + cfg.d_rope)) if prefix_latent is None else f64(prefix_latent)
    n_pre = pre.shape[0]
    pos = pos_offset + np.arange(T)
    cbar_l, kR_l = kv_latent(x, W["W_aKV"], gkv, pos, cfg)
    cbar = np.concatenate([pre[:, : cfg.kv_rank], cbar_l], 0)
    kR = np.concatenate([pre[:, cfg.kv_rank:], kR_l], 0)
    KC, V = kv_heads(cbar, W["W_bKV"], cfg)
    cQ, qC, qR = query_path(x, W["W_aQ"], W["W_bQ"], gq, pos, cfg)
    lam = lambda_coeff(x, W["W_lambda"])
    G = gate_logits(cQ, W["W_G"], cfg)
    first = pos_offset - n_pre           # position of key row 0
    y = np.empty((T, cfg.d_model))
    for t in range(T):
        lo, hi = key_range(int(pos[t]), cfg.window)
        lo = max(lo, first)
        H = attend_row(qC[t], qR[t], KC, kR, V, lo - first, hi - first, cfg)
        _, y[t] = combine_row(H, lam[t], G[t], W["W_O"], cfg)
    return y


def attention_stage(qC, qR, KC, V, kR, lam, G, cfg: OracleConfig):
    """The attention stage of one sequence on its projected inputs (section 2.2 of the picx.dev
    page: attention per head, D = H_S - lambda Repeat_g(H_N), sigmoid(G) gate).

    qC [T, n_H, d_nope], qR [T, n_H, d_rope] (rotated), KC [T, n_KV, d_nope], V [T, n_KV, d_v],
    kR [T, d_rope] (rotated), lam [T, n_S] (already sigmoided), G [T, n_S, d_v] (logits).
    Returns (Dg [T, n_S, d_v], H [T, n_H, d_v]).
    """
    T = qC.shape[0]
    H = np.empty((T, cfg.n_heads, cfg.d_v))
    for t in range(T):
        lo, hi = key_range(t, cfg.window)
        H[t] = attend_row(qC[t], qR[t], KC, kR, V, lo, hi, cfg)
    nmap = noise_of_signal(cfg)
    Dg = np.empty((T, cfg.n_signal, cfg.d_v))
    for t in range(T):
        _, Dg[t] = differential_combine(H[t, : cfg.n_signal], H[t, cfg.n_signal:], lam[t], G[t], nmap)
    return Dg, H


def attention_stage_backward(qC, qR, KC, V, kR, lam, G, dDg, cfg: OracleConfig):
    """Gradient of sum(dDg * Dg) with respect to every input of attention_stage.

    Written out from the definition by the chain rule: with g = sigmoid(G), D = H_S - lambda H_N,
      dG = dDg g (1 - g) D,  dH_S = dDg g,  dlambda_s = -sum_c dH_S[c] H_N(s)[c],
      dH_N(n) = -sum_{s -> n} lambda_s dH_S,
    and for each head's softmax attention H = P V, P = softmax(s), s = scale q.k:
      dV += P^T dH,  dP = dH V^T,  ds = P (dP - sum_k P dP) = P (dP - dH.H),
      dq = scale ds K,  dK += scale ds^T q  (K = [K^C ; k^R], q = [q^C ; q^R]).
    Returns a dict of dqC, dqR, dKC, dV, dkR, dlam, dG (same shapes as the inputs).
    """
    T = qC.shape[0]
    scale = 1.0 / np.sqrt(cfg.d_nope + cfg.d_rope)
    _, H = attention_stage(qC, qR, KC, V, kR, lam, G, cfg)
    nmap = noise_of_signal(cfg)
    kvh = kv_head_of(cfg)
    g = sigmoid(G)
    HS, HN = H[:, : cfg.n_signal], H[:, cfg.n_signal:]
    D = HS - lam[..., None] * HN[:, nmap]
    out = {k: np.zeros_like(v) for k, v in dict(dqC=qC, dqR=qR, dKC=KC, dV=V, dkR=kR).items()}
    out["dG"] = dDg * g * (1.0 - g) * D
    dHS = dDg * g
    out["dlam"] = -np.einsum("tsc,tsc->ts", dHS, HN[:, nmap])
    dH = np.zeros_like(H)
    dH[:, : cfg.n_signal] = dHS
    for s_ in range(cfg.n_signal):
        dH[:, cfg.n_signal + nmap[s_]] -= lam[:, s_, None] * dHS[:, s_]
    for t in range(T):
        lo, hi = key_range(t, cfg.window)
        for h in range(cfg.n_heads):
            j = kvh[h]
            k = np.concatenate([KC[lo: hi + 1, j], kR[lo: hi + 1]], -1)
            q = np.concatenate([qC[t, h], qR[t, h]])
            sc = (k @ q) * scale
            p = np.exp(sc - sc.max())
            p /= p.sum()
            dP = V[lo: hi + 1, j] @ dH[t, h]
            ds = p * (dP - dH[t, h] @ H[t, h])
            out["dV"][lo: hi + 1, j] += np.outer(p, dH[t, h])
            dq = scale * (ds @ k)
            out["dqC"][t, h] += dq[: cfg.d_nope]
            out["dqR"][t, h] += dq[cfg.d_nope:]
            dk = scale * np.outer(ds, q)
            out["dKC"][lo: hi + 1, j] += dk[:, : cfg.d_nope]
            out["dkR"][lo: hi + 1] += dk[:, cfg.d_nope:]
    return out


def attention_stage_backward_group(qC, qR, KC, V, kR, lam, G, dDg, cfg: OracleConfig, j: int,
                                   q_rows, k_rows, block: int = 512):
    """The part of attention_stage_backward that belongs to KV group j, at chosen rows.

    Returns dq^C, dq^R of the group's heads (its noise head and the signal heads that subtract
    it) at query rows q_rows; dK^C_j and dV_j at key rows k_rows; dlambda and dG of those signal
    heads at q_rows.  Same chain rule as attention_stage_backward; every query row's softmax
    statistics (the normaliser and H) are formed exactly, one block of rows at a time, so that
    long sequences need O(T^2) work for one group only.  Keys: dict with arrays "dqC" [len(q_rows),
    heads, d_nope], "dqR", "dKC" [len(k_rows), d_nope], "dV", "dlam" [len(q_rows), signals], "dG",
    and the head order "heads" (noise head first) and "signals".
    """
    T = qC.shape[0]
    scale = 1.0 / np.sqrt(cfg.d_nope + cfg.d_rope)
    nmap = noise_of_signal(cfg)
    signals = [s for s in range(cfg.n_signal) if nmap[s] == j]
    heads = [cfg.n_signal + j] + signals
    k = np.concatenate([KC[:, j], kR], -1)              # [T, 192]
    v = V[:, j]                                          # [T, d_v]
    # dH of every row needs only that row's inputs
    g = sigmoid(G[:, signals])
    dHS = dDg[:, signals] * g
    dH = {cfg.n_signal + j: -np.einsum("ts,tsc->tc", lam[:, signals], dHS)}
    for i, s_ in enumerate(signals):
        dH[s_] = dHS[:, i]
    # forward statistics of the group's heads over all query rows
    logZ = {h: np.empty(T) for h in heads}
    Hh = {h: np.empty((T, cfg.d_v)) for h in heads}
    tt = np.arange(T)
    for r0 in range(0, T, block):
        r1 = min(T, r0 + block)
        rows = tt[r0:r1]
        lo = np.array([key_range(int(t), cfg.window)[0] for t in rows])
        allowed = (tt[None, :] <= rows[:, None]) & (tt[None, :] >= lo[:, None])
        for h in heads:
            q = np.concatenate([qC[r0:r1, h], qR[r0:r1, h]], -1)
            sc = np.where(allowed, (q @ k.T) * scale, -np.inf)
            m = sc.max(-1, keepdims=True)
            e = np.exp(sc - m)
            z = e.sum(-1, keepdims=True)
            logZ[h][r0:r1] = (m + np.log(z))[:, 0]
            Hh[h][r0:r1] = (e / z) @ v
    delta = {h: np.einsum("tc,tc->t", dH[h], Hh[h]) for h in heads}
    out = {"heads": heads, "signals": signals}
    # key rows: dV_j[s] = sum_h sum_t P_h[t, s] dH_h[t];  dK_j[s] = scale sum_h sum_t dS_h[t, s] q_h[t]
    dKC = np.zeros((len(k_rows), cfg.d_nope))
    dVk = np.zeros((len(k_rows), cfg.d_v))
    for i, s in enumerate(k_rows):
        vis = np.array([key_range(int(t), cfg.window)[0] <= s <= t for t in range(T)])
        for h in heads:
            q = np.concatenate([qC[:, h], qR[:, h]], -1)
            p = np.where(vis, np.exp((q @ k[s]) * scale - logZ[h]), 0.0)
            dVk[i] += p @ dH[h]
            ds = p * (dH[h] @ v[s] - delta[h])
            dKC[i] += scale * (ds @ q)[: cfg.d_nope]
    out["dKC"], out["dV"] = dKC, dVk
    # query rows: dq_h[t] = scale sum_s dS_h[t, s] k[s]; dlambda, dG from H_S, H_N of row t
    dqC = np.zeros((len(q_rows), len(heads), cfg.d_nope))
    dqR = np.zeros((len(q_rows), len(heads), cfg.d_rope))
    dlam = np.zeros((len(q_rows), len(signals)))
    dG = np.zeros((len(q_rows), len(signals), cfg.d_v))
    for i, t in enumerate(q_rows):
        lo, hi = key_range(int(t), cfg.window)
        for a, h in enumerate(heads):
            q = np.concatenate([qC[t, h], qR[t, h]])
            p = np.exp((k[lo: hi + 1] @ q) * scale - logZ[h][t])
            ds = p * (v[lo: hi + 1] @ dH[h][t] - delta[h][t])
            dq = scale * (ds @ k[lo: hi + 1])
            dqC[i, a], dqR[i, a] = dq[: cfg.d_nope], dq[cfg.d_nope:]
        HN = Hh[cfg.n_signal + j][t]
        for b_, s_ in enumerate(signals):
            dlam[i, b_] = -dHS[t, b_] @ HN
            gs = sigmoid(G[t, s_])
            dG[i, b_] = dDg[t, s_] * gs * (1.0 - gs) * (Hh[s_][t] - lam[t, s_] * HN)
    out.update(dqC=dqC, dqR=dqR, dlam=dlam, dG=dG)
    return out


def gdla_prefill_packed(x_packed, cu_seqlens, weights: dict, cfg: OracleConfig, g_q=None, g_kv=None):
    """Packed documents: document d = rows cu[d] .. cu[d+1]-1 of x_packed [total, d_model] is an
    independent sequence (its own positions from 0, attention inside the document only).
    Returns y [total, d_model] in packed order."""
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    out = np.empty((cu[-1], cfg.d_model))
    for d in range(len(cu) - 1):
        if cu[d + 1] > cu[d]:
            out[cu[d]: cu[d + 1]] = gdla_prefill(x_packed[None, cu[d]: cu[d + 1]], weights, cfg,
                                                  g_q=g_q, g_kv=g_kv)[0]
    return out


# --------------------------------------------------------------------------------------
# full layer: decode (one new token per sequence, keys = cached latent rows + itself)
# --------------------------------------------------------------------------------------
def _decode_common(x_new, weights, cache, cache_len, cfg, g_q, g_kv, own_rows=None):
    """own_rows [B, kv_rank + d_rope]: the new tokens' latent rows as the cache stores them
    (e.g. after quantization), used as their own keys instead of the computed rows."""
    W = _weights64(weights)
    gq = None if g_q is None else f64(g_q)
    gkv = None if g_kv is None else f64(g_kv)
    xn = f64(x_new)
    lens = [int(v) for v in (cache_len.tolist() if hasattr(cache_len, "tolist") else cache_len)]
    pos = np.asarray(lens)
    cQ, qC, qR = query_path(xn, W["W_aQ"], W["W_bQ"], gq, pos, cfg)
    cbar_new, kR_new = kv_latent(xn, W["W_aKV"], gkv, pos, cfg)
    lam = lambda_coeff(xn, W["W_lambda"])
    G = gate_logits(cQ, W["W_G"], cfg)
    if own_rows is not None:
        own = f64(own_rows)
        cbar_new, kR_new = own[:, : cfg.kv_rank], own[:, cfg.kv_rank:]
    return W, lens, cQ, qC, qR, cbar_new, kR_new, lam, G


def _keys_of(cache, b, p, cbar_new, kR_new, cfg):
    """Latent rows 0..p of sequence b: the p cached rows followed by the new token's row."""
    rows = f64(cache[b, :p]) if p else np.zeros((0, cfg.kv_rank + cfg.d_rope))
    cbar = np.concatenate([rows[:, : cfg.kv_rank], cbar_new[b][None]], axis=0)
    kR = np.concatenate([rows[:, cfg.kv_rank:], kR_new[b][None]], axis=0)
    return cbar, kR


def gdla_decode(x_new, weights: dict, cache, cache_len, cfg: OracleConfig, g_q=None, g_kv=None,
                return_parts: bool = False, own_rows=None):
    """Literal decode: the prefill definition applied to the new token at position cache_len[b].

    cache [B, cap, kv_rank + d_rope] holds (normalised c^KV | rotated k^R) per cached token.
    K^C and V are re-expanded from the latent rows with W_bKV exactly as in prefill.
    Returns y [B, d] (and the new latent rows when ``return_parts``).
    """
    W, lens, cQ, qC, qR, cbar_new, kR_new, lam, G = _decode_common(
        x_new, weights, cache, cache_len, cfg, g_q, g_kv, own_rows)
    y = np.empty((len(lens), cfg.d_model))
    Dgs = []
    for b, p in enumerate(lens):
        cbar, kR = _keys_of(cache, b, p, cbar_new, kR_new, cfg)
        KC, V = kv_heads(cbar, W["W_bKV"], cfg)
        lo, hi = key_range(p, cfg.window)
        H = attend_row(qC[b], qR[b], KC, kR, V, lo, hi, cfg)
        Dg, y[b] = combine_row(H, lam[b], G[b], W["W_O"], cfg)
        Dgs.append(Dg)
    if return_parts:
        return y, dict(cbar_new=cbar_new, kR_new=kR_new, Dg=np.stack(Dgs), lam=lam, G=G)
    return y


def gdla_decode_absorbed(x_new, weights: dict, cache, cache_len, cfg: OracleConfig, g_q=None,
                         g_kv=None, own_rows=None):
    """Weight-absorbed decode: attention runs in the latent space, K^C and V are never formed.

    With W_UK_j / W_UV_j the K^C / V column blocks of W_bKV for KV head j:
      score_{h,s} = (W_UK_j q^C_h) . c_bar_s + q^R_h . k^R_s            (q^C_h . K^C_{j,s} regrouped)
      l_h        = sum_s p_{h,s} c_bar_s                               (latent attention output)
      D_s        = (l_s - lambda_s l_{n(s)}) W_UV_j                    (H = l W_UV, linear in l)
    Same result as ``gdla_decode`` up to rounding order; used for sizes where re-expanding
    every cached row is too slow.
    """
    W, lens, cQ, qC, qR, cbar_new, kR_new, lam, G = _decode_common(
        x_new, weights, cache, cache_len, cfg, g_q, g_kv, own_rows)
    scale = 1.0 / np.sqrt(cfg.d_nope + cfg.d_rope)
    kvh = kv_head_of(cfg)
    nmap = noise_of_signal(cfg)
    blk = cfg.d_nope + cfg.d_v
    W_UK = [W["W_bKV"][:, j * blk: j * blk + cfg.d_nope] for j in range(cfg.n_kv_heads)]
    W_UV = [W["W_bKV"][:, j * blk + cfg.d_nope: (j + 1) * blk] for j in range(cfg.n_kv_heads)]
    y = np.empty((len(lens), cfg.d_model))
    for b, p in enumerate(lens):
        cbar, kR = _keys_of(cache, b, p, cbar_new, kR_new, cfg)
        lo, hi = key_range(p, cfg.window)
        cbar, kR = cbar[lo: hi + 1], kR[lo: hi + 1]
        qt = np.stack([W_UK[kvh[h]] @ qC[b, h] for h in range(cfg.n_heads)])   # [n_H, kv_rank]
        s = (qt @ cbar.T + qR[b] @ kR.T) * scale
        s = s - s.max(axis=-1, keepdims=True)
        pr = np.exp(s)
        pr = pr / pr.sum(axis=-1, keepdims=True)
        lat = pr @ cbar                                                          # [n_H, kv_rank]
        lat_S, lat_N = lat[: cfg.n_signal], lat[cfg.n_signal:]
        Dlat = lat_S - lam[b][:, None] * lat_N[nmap]
        D = np.stack([Dlat[s_] @ W_UV[kvh[s_]] for s_ in range(cfg.n_signal)])
        Dg = sigmoid(G[b]) * D
        y[b] = Dg.reshape(-1) @ W["W_O"]
    return y


def gdla_decode_multi(x_new, weights: dict, cache, cache_len, cfg: OracleConfig, g_q=None, g_kv=None,
                      route: str = "literal"):
    """q_len new tokens per sequence: x_new [B, q_len, d].  Token i of sequence b is at position
    cache_len[b] + i and sees the cached rows plus new tokens 0..i; this is q_len consecutive
    single-token decodes, each over the cache extended by the earlier new tokens' latent rows
    (computed here in float64).  route selects the literal or the weight-absorbed decode.
    Returns y [B, q_len, d]."""
    W = _weights64(weights)
    gkv = None if g_kv is None else f64(g_kv)
    one = gdla_decode if route == "literal" else gdla_decode_absorbed
    xn = f64(x_new)
    B, q = xn.shape[0], xn.shape[1]
    lens = [int(v) for v in (cache_len.tolist() if hasattr(cache_len, "tolist") else cache_len)]
    y = np.empty((B, q, cfg.d_model))
    for b in range(B):
        L = lens[b]
        rows = f64(cache[b, :L]) if L else np.zeros((0, cfg.kv_rank + cfg.d_rope))
        cbar, kR = kv_latent(xn[b], W["W_aKV"], gkv, L + np.arange(q), cfg)
        ext = np.concatenate([rows, np.concatenate([cbar, kR], -1)], 0)[None]
        for i in range(q):
            y[b, i] = one(xn[b, i][None], weights, ext, [L + i], cfg, g_q=g_q, g_kv=g_kv)[0]
    return y


# --------------------------------------------------------------------------------------
# MXFP8 latent cache: decode over cache rows stored at 8 bits per value
# --------------------------------------------------------------------------------------
# The report's low-precision recipe stores tensors in MXFP8 (paperglide.net summary, the
# low-precision training paragraph and the Figure 3 caption).  Written out here from the
# format's definition (OCP microscaling: blocks of 32 values sharing one power-of-two scale,
# stored as an 8-bit exponent E with scale 2^(E - 127); values in FP8 E4M3):
#   E4M3 byte s.eeee.mmm: e = 0 -> (-1)^s 2^-6 (m / 8) (zero and subnormals); e > 0 ->
#   (-1)^s 2^(e - 7) (1 + m / 8); s.1111.111 is NaN; no infinities; largest finite 448.
# Readings where the pages say nothing (listed in the design notes):
#   * a latent-cache row (576 values: normalised c^KV | rotated k^R) is 18 blocks of 32;
#   * the block scale is the smallest power of two 2^k with max|v| <= 448 2^k (nothing is
#     clipped), k in [-127, 127]; an all-zero block takes k = -127;
#   * values v / 2^k are rounded to the nearest E4M3 value, ties to the even code;
#   * a row of n values (n a multiple of 32) is stored as n E4M3 bytes, then its n / 32 scale
#     bytes, then zero bytes up to a multiple of 16: 576 + 18 + 14 = 608 bytes for the layer's rows.
FP8_BLOCK = 32
E4M3_MAX = 448.0


def fp8_row_bytes(n: int) -> int:
    """Stored bytes of a row of n values."""
    return (n + n // FP8_BLOCK + 15) // 16 * 16


def e4m3_value(codes) -> np.ndarray:
    """float64 value of E4M3 codes (NaN for the two NaN codes), from the bit fields."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_value(np.arange(0x7F))          # codes 0x00..0x7E: the finite values >= 0, increasing


def e4m3_round(x) -> np.ndarray:
    """Codes of the E4M3 values nearest to finite x (ties to the even code), saturating at
    +-448.  By search over the 127 non-negative finite values; the sign bit is x's sign (the
    format is sign-magnitude: a negative x that rounds to zero gives -0, code 0x80)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 0x7E)       # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - _E4M3_POS[lo], _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a == _E4M3_POS[hi], hi, code)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def mx_block_exponent(amax) -> np.ndarray:
    """Smallest k with amax <= 448 * 2^k (k in [-127, 127]); -127 for an all-zero block."""
    amax = np.asarray(amax, dtype=np.float64)
    out = np.full(amax.shape, -127, dtype=np.int64)
    nz = amax > 0
    k = np.ceil(np.log2(np.where(nz, amax, 1.0) / E4M3_MAX)).astype(np.int64)
    # log2 is a library routine with rounding: settle the boundary exactly
    k = np.where(E4M3_MAX * np.exp2(k.astype(np.float64)) < amax, k + 1, k)
    k = np.where(E4M3_MAX * np.exp2((k - 1).astype(np.float64)) >= amax, k - 1, k)
    out[nz] = np.clip(k[nz], -127, 127)
    return out


def mxfp8_quantize_rows(rows) -> np.ndarray:
    """Rows [N, n] (any float values; n a multiple of 32) -> stored bytes [N, fp8_row_bytes(n)]."""
    v = f64(rows)
    v = v.reshape(-1, v.shape[-1])
    n = v.shape[1]
    blk = v.reshape(v.shape[0], -1, FP8_BLOCK)
    k = mx_block_exponent(np.abs(blk).max(axis=-1))                     # [N, n / 32]
    q = e4m3_round(blk / np.exp2(k.astype(np.float64))[..., None]).reshape(v.shape[0], n)
    out = np.zeros((v.shape[0], fp8_row_bytes(n)), dtype=np.uint8)
    out[:, :n] = q
    out[:, n: n + k.shape[1]] = (k + 127).astype(np.uint8)
    return out


def mxfp8_dequantize_rows(stored, n: int) -> np.ndarray:
    """Stored bytes [N, fp8_row_bytes(n)] -> float64 rows [N, n]: each E4M3 value times its
    block's 2^(E - 127)."""
    b = np.asarray(stored, dtype=np.uint8).reshape(-1, fp8_row_bytes(n))
    nblk = n // FP8_BLOCK
    vals = e4m3_value(b[:, :n]).reshape(b.shape[0], nblk, FP8_BLOCK)
    k = b[:, n: n + nblk].astype(np.int64) - 127
    return (vals * np.exp2(k.astype(np.float64))[..., None]).reshape(b.shape[0], n)


def gdla_decode_fp8(x_new, weights: dict, cache8, cache_len, cfg: OracleConfig, g_q=None, g_kv=None,
                    route: str = "absorbed", q_len: int = 1):
    """Decode over an MXFP8 latent cache cache8 [B, cap, fp8_row_bytes(kv_rank + d_rope)] (uint8).  Every key row the
    attention reads is the dequantized stored row, the new tokens' own rows included: each new
    token's latent row is rounded to bf16 and quantized (it is what the cache receives) and read
    back.  With q_len > 1,
    x_new is [B, q_len, d] and token i sits at position cache_len[b] + i.  Returns y [B, q_len, d]
    (q_len > 1) or [B, d]."""
    W = _weights64(weights)
    gkv = None if g_kv is None else f64(g_kv)
    one = gdla_decode if route == "literal" else gdla_decode_absorbed
    xn = f64(x_new)
    one_token = q_len == 1 and xn.ndim == 2
    if one_token:
        xn = xn[:, None, :]
    B, q = xn.shape[0], xn.shape[1]
    lens = [int(v) for v in (cache_len.tolist() if hasattr(cache_len, "tolist") else cache_len)]
    y = np.empty((B, q, cfg.d_model))
    for b in range(B):
        L = lens[b]
        n = cfg.kv_rank + cfg.d_rope
        rows = mxfp8_dequantize_rows(np.asarray(cache8[b, :L]), n) if L else np.zeros((0, n))
        cbar, kR = kv_latent(xn[b], W["W_aKV"], gkv, L + np.arange(q), cfg)
        # what the cache receives: the MXFP8 form of the bf16 latent values (the row a bf16
        # cache would hold; rounding to bf16 is a library step)
        import torch
        lat_bf16 = torch.tensor(np.concatenate([cbar, kR], -1)).to(torch.bfloat16).double().numpy()
        new = mxfp8_dequantize_rows(mxfp8_quantize_rows(lat_bf16), n)
        ext = np.concatenate([rows, new], 0)[None]
        for i in range(q):
            # keys: the cached rows, the earlier new tokens' stored rows, and its own stored row
            y[b, i] = one(xn[b, i][None], weights, ext, [L + i], cfg, g_q=g_q, g_kv=g_kv,
                          own_rows=ext[0, L + i][None])[0]
    return y[:, 0] if one_token else y
