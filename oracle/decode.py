"""fp64 oracle for one decode step of attention over a KV cache — TEST
INFRASTRUCTURE ONLY (same rules as the rest of ``oracle``).

Source: apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour 50€ ?",
§ "Comment nanochat fonctionne" › 6 "Moteur d'inférence": the engine keeps a
KV cache filled at prefill and generates one token per sequence per step,
through the same causal, windowed, grouped-query attention as training (§ 5,
flash_attn_func(q, k, v, causal=True, window_size=...)).

Reading (also in the design notes): at a decode step the cache of sequence b
holds positions 0 .. lens[b]-1, the new token's own k and v included; the new
token sits at position lens[b]-1 and sees the same keys its row of the
training-time attention sees: lens[b]-1-W .. lens[b]-1 (all when W < 0).
"""
import numpy as np


def decode_attention(q, k_cache, v_cache, lens, window):
    """q [B,H,hd]; k_cache, v_cache [B,Tmax,Hkv,hd]; lens [B] -> o [B,H,hd], lse [B,H]."""
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    B, H, hd = q.shape
    Hk = k_cache.shape[2]
    G = H // Hk
    scale = 1.0 / np.sqrt(hd)
    o = np.zeros((B, H, hd))
    lse = np.zeros((B, H))
    for b in range(B):
        t = int(lens[b]) - 1
        lo = max(0, t - window) if window is not None and window >= 0 else 0
        for h in range(H):
            kv = h // G
            s = (k_cache[b, lo:t + 1, kv, :] @ q[b, h, :]) * scale
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            o[b, h, :] = (e / z) @ v_cache[b, lo:t + 1, kv, :]
            lse[b, h] = m + np.log(z)
    return o, lse
