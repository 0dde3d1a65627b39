"""An independent second statement of the action expert in PyTorch (CPU, float64).

Used only to cross-check the oracle.  It is written in a different style on
purpose -- all suffixes batched, torch.nn.functional's rms_norm / gelu /
silu / scaled_dot_product_attention with an explicit boolean mask, a
complex-number RoPE -- so that a slip in one statement (a transposed
operand, a dropped term, a wrong pairing) shows up as a disagreement.
"""

from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

T64 = torch.float64


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=T64)


def time_cond(W, t, width):
    half = width // 2
    expo = torch.linspace(0.0, 1.0, half, dtype=T64)
    period = 4e-3 * torch.pow(torch.tensor(4.0 / 4e-3, dtype=T64), expo)
    ang = 2 * math.pi * t / period
    e = torch.cat([torch.sin(ang), torch.cos(ang)])
    z = F.linear(e, _t(W["time_mlp_in.w"]), _t(W["time_mlp_in.b"]))
    return F.linear(F.silu(z), _t(W["time_mlp_out.w"]), _t(W["time_mlp_out.b"]))


def rope_complex(x, pos, theta):
    """x [..., S, heads, D]; rotate pairs (d, d+D/2) as complex numbers d + i(d+D/2)."""
    if theta == 0:
        return x
    d = x.shape[-1]
    half = d // 2
    freqs = 1.0 / (theta ** (torch.arange(0, half, dtype=T64) * 2.0 / d))
    ang = pos.to(T64)[:, None] * freqs[None, :]            # [S, half]
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]  # [S, 1, half]
    z = torch.complex(x[..., :half], x[..., half:]) * rot
    return torch.cat([z.real, z.imag], dim=-1)


def velocity(W, cfg, x_t, state, t, prefix_k, prefix_v):
    """v [G][H][A] for G suffixes sharing one prefix; t is a per-suffix sequence.

    x_t [G][H][A], state [Sd], prefix_k/v [L][P][Hkv][D]."""
    x_t = _t(x_t)
    g_count, h_len, _ = x_t.shape
    s_len = h_len + 1
    p_len = prefix_k.shape[1]
    hq, hkv, d = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    w = cfg.width
    eps = cfg.rms_eps

    tc = getattr(cfg, "time_cond", "add")
    st = F.linear(_t(state), _t(W["state_proj.w"]), _t(W["state_proj.b"]))
    act = F.linear(x_t, _t(W["action_in_proj.w"]), _t(W["action_in_proj.b"]))
    if tc == "concat":
        emb = []
        for g in range(g_count):
            half = w // 2
            expo = torch.linspace(0.0, 1.0, half, dtype=T64)
            period = 4e-3 * torch.pow(torch.tensor(4.0 / 4e-3, dtype=T64), expo)
            ang = 2 * math.pi * float(t[g]) / period
            e = torch.cat([torch.sin(ang), torch.cos(ang)]).expand(h_len, w)
            z = F.linear(torch.cat([act[g], e], dim=-1), _t(W["time_mlp_in.w"]), _t(W["time_mlp_in.b"]))
            emb.append(F.linear(F.silu(z), _t(W["time_mlp_out.w"]), _t(W["time_mlp_out.b"])))
        tokens = torch.stack(emb)
        c = None
    else:
        c = torch.stack([time_cond(W, float(tt), w) for tt in t])      # [G, w]
        tokens = act + c[:, None, :] if tc == "add" else act
    h = torch.cat([st.expand(g_count, 1, w), tokens], dim=1)  # [G, S, w]

    pos = torch.arange(p_len, p_len + s_len)
    mask = torch.ones(s_len, p_len + s_len, dtype=torch.bool)
    if cfg.suffix_mask == "pi0_block":
        mask[0, p_len + 1:] = False

    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        if tc == "adarms":
            mod = F.linear(c, _t(W[p + "time_mod.w"]), _t(W[p + "time_mod.b"]))[:, None, :]   # [G, 1, 6w]
            sa, ba, ga, sm, bm, gm = torch.chunk(mod, 6, dim=-1)
            u = F.rms_norm(h, (w,), eps=eps) * (1.0 + sa) + ba
        else:
            u = F.rms_norm(h, (w,), weight=1.0 + _t(W[p + "attn_norm.g"]), eps=eps)
        q = F.linear(u, _t(W[p + "q_proj.w"])).view(g_count, s_len, hq, d)
        k = F.linear(u, _t(W[p + "k_proj.w"])).view(g_count, s_len, hkv, d)
        v = F.linear(u, _t(W[p + "v_proj.w"])).view(g_count, s_len, hkv, d)
        q = rope_complex(q, pos, cfg.rope_theta)
        k = rope_complex(k, pos, cfg.rope_theta)
        pk = _t(prefix_k[l]).expand(g_count, p_len, hkv, d)
        pv = _t(prefix_v[l]).expand(g_count, p_len, hkv, d)
        keys = torch.cat([pk, k], dim=1).transpose(1, 2)     # [G, Hkv, keys, D]
        vals = torch.cat([pv, v], dim=1).transpose(1, 2)
        rep = hq // hkv
        keys = keys.repeat_interleave(rep, dim=1)
        vals = vals.repeat_interleave(rep, dim=1)
        o = F.scaled_dot_product_attention(q.transpose(1, 2), keys, vals, attn_mask=mask)
        o = o.transpose(1, 2).reshape(g_count, s_len, hq * d)
        if tc == "adarms":
            h = h + ga * F.linear(o, _t(W[p + "o_proj.w"]))
            u = F.rms_norm(h, (w,), eps=eps) * (1.0 + sm) + bm
        else:
            h = h + F.linear(o, _t(W[p + "o_proj.w"]))
            u = F.rms_norm(h, (w,), weight=1.0 + _t(W[p + "mlp_norm.g"]), eps=eps)
        gate = F.gelu(F.linear(u, _t(W[p + "gate_proj.w"])), approximate="tanh")
        branch = F.linear(gate * F.linear(u, _t(W[p + "up_proj.w"])), _t(W[p + "down_proj.w"]))
        h = h + (gm * branch if tc == "adarms" else branch)

    hf = F.rms_norm(h[:, 1:], (w,), weight=1.0 + _t(W["final_norm.g"]), eps=eps)
    return F.linear(hf, _t(W["action_out_proj.w"]), _t(W["action_out_proj.b"])).numpy()


def draft(W, dcfg, vis):
    """Candidate chunks [B][H][A] of the FLASH draft model for vis [B][V][w]:
    the queries are concatenated after the visual tokens of every batch
    element and one block runs over the batched sequences."""
    vis = _t(vis)
    b, v_len, w = vis.shape
    h_len = dcfg.n_queries
    n = v_len + h_len
    hq, hkv, d = dcfg.n_q_heads, dcfg.n_kv_heads, dcfg.head_dim
    eps = dcfg.rms_eps
    x = torch.cat([vis, _t(W["action_queries"]).expand(b, h_len, w)], dim=1)     # [B, n, w]
    pos = torch.arange(n)
    u = F.rms_norm(x, (w,), weight=1.0 + _t(W["attn_norm.g"]), eps=eps)
    q = rope_complex(F.linear(u, _t(W["q_proj.w"])).view(b, n, hq, d), pos, dcfg.rope_theta)
    k = rope_complex(F.linear(u, _t(W["k_proj.w"])).view(b, n, hkv, d), pos, dcfg.rope_theta)
    v = F.linear(u, _t(W["v_proj.w"])).view(b, n, hkv, d)
    rep = hq // hkv
    o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2).repeat_interleave(rep, dim=1),
                                       v.transpose(1, 2).repeat_interleave(rep, dim=1))
    h = x + F.linear(o.transpose(1, 2).reshape(b, n, hq * d), _t(W["o_proj.w"]))
    u = F.rms_norm(h, (w,), weight=1.0 + _t(W["mlp_norm.g"]), eps=eps)
    gate = F.gelu(F.linear(u, _t(W["gate_proj.w"])), approximate="tanh")
    h = h + F.linear(gate * F.linear(u, _t(W["up_proj.w"])), _t(W["down_proj.w"]))
    return F.linear(h[:, v_len:], _t(W["action_head.w"]), _t(W["action_head.b"])).numpy()


def prefill_kv(W, pcfg, emb):
    """KV cache [L][2][1][P][Hkv][D] of the prefill stack over emb [P][w];
    the whole prefix attends to itself without a mask."""
    h = _t(emb)[None]                       # [1, P, w]
    p_len, w = h.shape[1], h.shape[2]
    hq, hkv, d = pcfg.n_q_heads, pcfg.n_kv_heads, pcfg.head_dim
    pos = torch.arange(p_len)
    out = torch.zeros(pcfg.n_layers, 2, 1, p_len, hkv, d, dtype=T64)
    for l in range(pcfg.n_layers):
        p = f"layers.{l}."
        u = F.rms_norm(h, (w,), weight=1.0 + _t(W[p + "attn_norm.g"]), eps=pcfg.rms_eps)
        k = rope_complex(F.linear(u, _t(W[p + "k_proj.w"])).view(1, p_len, hkv, d), pos, pcfg.rope_theta)
        v = F.linear(u, _t(W[p + "v_proj.w"])).view(1, p_len, hkv, d)
        out[l, 0] = k
        out[l, 1] = v
        q = rope_complex(F.linear(u, _t(W[p + "q_proj.w"])).view(1, p_len, hq, d), pos, pcfg.rope_theta)
        rep = hq // hkv
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2).repeat_interleave(rep, dim=1),
                                           v.transpose(1, 2).repeat_interleave(rep, dim=1))
        h = h + F.linear(o.transpose(1, 2).reshape(1, p_len, hq * d), _t(W[p + "o_proj.w"]))
        u = F.rms_norm(h, (w,), weight=1.0 + _t(W[p + "mlp_norm.g"]), eps=pcfg.rms_eps)
        gate = F.gelu(F.linear(u, _t(W[p + "gate_proj.w"])), approximate="tanh")
        h = h + F.linear(gate * F.linear(u, _t(W[p + "up_proj.w"])), _t(W[p + "down_proj.w"]))
    return out.numpy()
