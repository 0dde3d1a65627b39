"""Oracle: a plain, slow, fp64 CPU statement of the flow-matching action-expert
suffix loop and of FLASH parallel verification.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The product package never imports it and shares no code with it; the only
common dependency is the seeded input generator in ``synthetic/``.

Every function below follows one passage of the pages, cited by page title
and section:

  [DM0.5]  "DM0.5: high-performance embodied VLA and OpenDM reading guide"
           sec. 5.1 (prefix encoded once into a per-layer KV cache),
           sec. 5.2 (action expert: action_in_proj, time_mlp_in/out, prefix
           KV access, action_out_proj -> velocity), sec. 5.3 (flow matching:
           x_t = t*eps + (1-t)*a, u_t = eps - a, Euler sampling from noise,
           diffusion_steps = 10, action chunk), sec. 6.3 (MLP = gate/up/down).
  [FLASH]  "Realtime-VLA FLASH: speculative inference for diffusion VLAs"
           sec. 02 (interpolate the draft with noise at several times,
           predict velocities in parallel, rebuild endpoints, compare with
           the draft), sec. 03.2 (accept a prefix whose distance is below
           delta at every verification time; zero accepted length -> full
           path), sec. 03.3 (a gripper switch in the candidate chunk forces
           the full path).
  [RTVLA]  "Running VLAs at Real-time Speed": 10 iterations of tens of layers.

Pins: every elementary function is pinned in tests/test_oracle_pins.py
against closed forms, brute force or library routines.  expert_velocity
(the composed random-weight expert): parity unpinned by the pages, which
print no worked numerical example; it is pinned only through its parts, the
zero-layer closed form and an independent PyTorch restatement.

Where the pages are silent the plainest reading is taken:
  R1 Euler sign: x <- x - dt*v with dt = 1/N, t_k = 1 - k/N (integrating from
     noise at t=1 to data at t=0 under u = eps - a).
  R2 time conditioning: c = W_to . swish(W_ti . e(t) + b_ti) + b_to added to
     every action token; e(t) = [sin(2 pi t / p_i), cos(2 pi t / p_i)] with
     p_i geometric from 4e-3 to 4.0.
  R3 suffix mask: every suffix token sees all prefix tokens and all tokens of
     its own suffix ("bidir"); "pi0_block" hides the action rows from the
     state row.
  R4 RoPE on suffix q/k at positions P..P+S-1, half-split pairs, theta 1e4;
     prefix keys are given already rotated.
  R5 RMSNorm x / sqrt(mean(x^2) + eps) * (1 + g), eps = 1e-6; a final norm
     precedes action_out_proj.
  R6 GELU tanh approximation in the gated MLP.
  R7 biases only on state_proj, action_in/out_proj and the time MLP.
  R8 only the H action rows produce velocity; the state row is discarded.
  R10 FP8 MLP (the pi0-fp8mlp workload; [DM0.5] 6.3 names FP8 E4M3 for the
     gate/up/down GEMMs): gate/up/down given as E4M3
     codes with one fp32 scale per output row; W = decode(code) * scale,
     everything else unchanged (bf16 activations, fp32 accumulation on the
     device; fp64 here).
  R16 Pi0 time conditioning (the pi0-concat workload; the "VLA design space"
     slides and [DM0.5] 5.2 name the time MLP without its form): an action
     token is W_to . swish(W_ti . [W_ai x + b_ai ; e(t)] + b_ti) + b_to, with
     e(t) of the model width as in R2 and W_ti of shape [w][2w]; nothing is
     added to it afterwards; the state token is unchanged.
  R17 DM0.5 per-layer time modulator ([DM0.5] 5.2 lists a time modulator in
     every layer and no formula; the dm05-adarms workload): the adaptive
     norm of the adaLN-Zero form (Peebles and Xie, "Scalable Diffusion
     Models with Transformers"): c(t) as in R2; per layer
     m = time_mod.w . c + time_mod.b, split into (scale_a, shift_a, gate_a,
     scale_m, shift_m, gate_m); each norm becomes
     x / rms(x) * (1 + scale) + shift on every suffix row and each branch's
     output is multiplied by its gate before the residual add; the final
     norm stays plain; c is not added to the tokens.  6 w^2 + 6 w
     parameters per layer (113M at width 1024 over 18 layers).
  R9 verify: per-row L2 distance over all action dims, strict d < delta,
     accepted length = longest prefix passing at every tau, one eps shared by
     all taus, gripper switch = sign (value > 0) change between consecutive
     draft rows anywhere in the chunk.
"""

from __future__ import annotations

from typing import Callable, Dict, Sequence, Tuple

import numpy as np

F64 = np.float64

# Sinusoid period range of the time embedding (reading R2).
MIN_PERIOD = 4e-3
MAX_PERIOD = 4.0

FLAG_ZERO_ACCEPT = 1      # accepted length is 0 -> full path      [FLASH] 03.2
FLAG_SWITCH = 2           # gripper switch inside the draft chunk  [FLASH] 03.3
FLAG_SWITCH_IN_PREFIX = 4  # a switch lies inside the accepted prefix


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Values of FP8 E4M3 codes ([DM0.5] sec. 6.3 names FP8 E4M3 for the MLP
    projections): bit 7 the sign, bits 6-3 the exponent with bias 7, bits 2-0
    the mantissa; exponent 0 holds the subnormals (m/8) * 2^-6, every other
    exponent (1 + m/8) * 2^(e-7); the code S.1111.111 is NaN and there are no
    infinities (largest finite value 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(F64)))
    return np.where((e == 15) & (m == 7), np.nan, sign * mag)


def to_f64(weights: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """fp64 values of the given parameters.  A matrix given as FP8 E4M3 codes
    (uint8) is decoded and multiplied row by row by its fp32 scale (the
    tensor of the same name ending in ".s"): the FP8 MLP storage,
    one scale per output channel."""
    out: Dict[str, np.ndarray] = {}
    for k, v in weights.items():
        if k.endswith(".s"):
            continue
        a = np.asarray(v)
        if a.dtype == np.uint8:
            out[k] = e4m3_decode(a) * np.asarray(weights[k[:-2] + ".s"], dtype=F64)[:, None]
        else:
            out[k] = a.astype(F64)
    return out


# ---------------------------------------------------------------------------
# elementary operations
# ---------------------------------------------------------------------------

def linear(x: np.ndarray, w: np.ndarray, b: np.ndarray | None = None) -> np.ndarray:
    """y = x . W^T (+ b) for W stored [out][in]."""
    y = np.matmul(x, w.T)
    if b is not None:
        y = y + b
    return y


def swish(z: np.ndarray) -> np.ndarray:
    """swish(z) = z * sigmoid(z) (the time MLP's activation, [DM0.5] 5.2)."""
    return z / (1.0 + np.exp(-z))


def gelu_tanh(z: np.ndarray) -> np.ndarray:
    """GELU, tanh approximation (reading R6)."""
    return 0.5 * z * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (z + 0.044715 * z ** 3)))


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """Gemma RMSNorm over the last axis with gain (1 + g) (reading R5)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * (1.0 + g)


def time_embedding(t: float, width: int) -> np.ndarray:
    """Sinusoidal embedding e(t) of the flow time, length ``width`` (reading R2)."""
    half = width // 2
    i = np.arange(half, dtype=F64)
    period = MIN_PERIOD * (MAX_PERIOD / MIN_PERIOD) ** (i / (half - 1))
    angle = 2.0 * np.pi * F64(t) / period
    return np.concatenate([np.sin(angle), np.cos(angle)])


def time_condition(W: Dict[str, np.ndarray], t: float) -> np.ndarray:
    """c(t) = time_mlp_out(swish(time_mlp_in(e(t))))   ([DM0.5] 5.2, reading R2)."""
    e = time_embedding(t, W["time_mlp_in.w"].shape[1])
    z = linear(e, W["time_mlp_in.w"], W["time_mlp_in.b"])
    return linear(swish(z), W["time_mlp_out.w"], W["time_mlp_out.b"])


def time_mlp_concat(W: Dict[str, np.ndarray], a: np.ndarray, t: float) -> np.ndarray:
    """Pi0's action-time MLP over [a ; e(t)] for action embeddings a [H][w] (reading R16)."""
    e = np.broadcast_to(time_embedding(t, a.shape[-1]), a.shape)
    z = linear(np.concatenate([a, e], axis=-1), W["time_mlp_in.w"], W["time_mlp_in.b"])
    return linear(swish(z), W["time_mlp_out.w"], W["time_mlp_out.b"])


def time_modulation(W: Dict[str, np.ndarray], l: int, c: np.ndarray):
    """Layer l's (scale_a, shift_a, gate_a, scale_m, shift_m, gate_m) from c(t) (reading R17)."""
    m = linear(c, W[f"layers.{l}.time_mod.w"], W[f"layers.{l}.time_mod.b"])
    return np.split(m, 6, axis=-1)


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding of x [S][heads][D] (reading R4).

    The pair (d, d + D/2) of a row at position p is rotated by the angle
    p * theta^(-2d/D).  theta == 0 turns the rotation off.
    """
    if theta == 0:
        return x
    d_model = x.shape[-1]
    half = d_model // 2
    inv_freq = F64(theta) ** (-2.0 * np.arange(half, dtype=F64) / d_model)
    ang = positions.astype(F64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def suffix_visibility(suffix_len: int, prefix_len: int, mode: str = "bidir") -> np.ndarray:
    """visible[r][j]: may suffix row r attend to key j of [prefix ; own suffix]?  (reading R3)"""
    vis = np.ones((suffix_len, prefix_len + suffix_len), dtype=bool)
    if mode == "pi0_block":
        vis[0, prefix_len + 1:] = False
    elif mode != "bidir":
        raise ValueError(mode)
    return vis


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, visible: np.ndarray) -> np.ndarray:
    """Grouped-query softmax attention ([DM0.5] 5.1/5.2, 6.2).

    q [S][Hq][D]; k, v [keys][Hkv][D]; visible [S][keys].  Query head j reads
    kv head floor(j * Hkv / Hq); scores are scaled by 1/sqrt(D); the softmax
    subtracts the row maximum.
    """
    s_len, hq, d = q.shape
    hkv = k.shape[1]
    out = np.zeros((s_len, hq, d), dtype=F64)
    for j in range(hq):
        kv = (j * hkv) // hq
        scores = np.matmul(q[:, j, :], k[:, kv, :].T) / np.sqrt(F64(d))
        scores = np.where(visible, scores, -np.inf)
        scores = scores - scores.max(axis=1, keepdims=True)
        p = np.exp(scores)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, j, :] = np.matmul(p, v[:, kv, :])
    return out


# ---------------------------------------------------------------------------
# the action expert: one velocity evaluation v_theta(x_t, t | c)
# ---------------------------------------------------------------------------

def expert_velocity(W: Dict[str, np.ndarray], cfg, x_t: np.ndarray, state: np.ndarray, t: float,
                    prefix_k: np.ndarray, prefix_v: np.ndarray) -> np.ndarray:
    """Velocity v [H][A] of one suffix ([DM0.5] 5.2; readings R2-R8).

    x_t [H][A]; state [Sd]; prefix_k / prefix_v [L][P][Hkv][D].
    """
    s_len = cfg.chunk_len + 1
    p_len = prefix_k.shape[1]
    hq, hkv, d = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    eps = cfg.rms_eps

    # suffix embedding: state token, then action tokens with the time
    # condition (added, R2; through Pi0's concat MLP, R16; or, R17, only
    # through the per-layer modulator)
    tc = getattr(cfg, "time_cond", "add")
    h = np.empty((s_len, cfg.width), dtype=F64)
    h[0] = linear(np.asarray(state, F64), W["state_proj.w"], W["state_proj.b"])
    a = linear(np.asarray(x_t, F64), W["action_in_proj.w"], W["action_in_proj.b"])
    c = time_condition(W, t) if tc != "concat" else None
    if tc == "add":
        h[1:] = a + c
    elif tc == "concat":
        h[1:] = time_mlp_concat(W, a, t)
    elif tc == "adarms":
        h[1:] = a
    else:
        raise ValueError(tc)

    positions = p_len + np.arange(s_len)
    visible = suffix_visibility(s_len, p_len, cfg.suffix_mask)
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        if tc == "adarms":
            sa, ba, ga, sm, bm, gm = time_modulation(W, l, c)
            u = rms_norm(h, sa, eps) + ba
        else:
            u = rms_norm(h, W[p + "attn_norm.g"], eps)
        q = linear(u, W[p + "q_proj.w"]).reshape(s_len, hq, d)
        k = linear(u, W[p + "k_proj.w"]).reshape(s_len, hkv, d)
        v = linear(u, W[p + "v_proj.w"]).reshape(s_len, hkv, d)
        q = rope(q, positions, cfg.rope_theta)
        k = rope(k, positions, cfg.rope_theta)
        keys = np.concatenate([prefix_k[l].astype(F64), k], axis=0)
        vals = np.concatenate([prefix_v[l].astype(F64), v], axis=0)
        o = attention(q, keys, vals, visible).reshape(s_len, hq * d)
        if tc == "adarms":
            h = h + ga * linear(o, W[p + "o_proj.w"])
            u = rms_norm(h, sm, eps) + bm
        else:
            h = h + linear(o, W[p + "o_proj.w"])
            u = rms_norm(h, W[p + "mlp_norm.g"], eps)
        m = gelu_tanh(linear(u, W[p + "gate_proj.w"])) * linear(u, W[p + "up_proj.w"])
        h = h + (gm if tc == "adarms" else 1.0) * linear(m, W[p + "down_proj.w"])

    hf = rms_norm(h[1:], W["final_norm.g"], eps)
    return linear(hf, W["action_out_proj.w"], W["action_out_proj.b"])


# ---------------------------------------------------------------------------
# denoising: N Euler steps from noise (t = 1) to the action chunk (t = 0)
# ---------------------------------------------------------------------------

def step_times(n_steps: int) -> np.ndarray:
    """t_k = 1 - k/N, k = 0..N-1 (reading R1)."""
    return 1.0 - np.arange(n_steps, dtype=F64) / F64(n_steps)


def euler_integrate(velocity: Callable[[np.ndarray, float], np.ndarray], noise: np.ndarray,
                    n_steps: int) -> np.ndarray:
    """x <- x - dt * v(x, t_k) for k = 0..N-1, dt = 1/N   ([DM0.5] 5.3, reading R1)."""
    x = np.asarray(noise, dtype=F64)
    dt = 1.0 / F64(n_steps)
    for t in step_times(n_steps):
        x = x - dt * velocity(x, float(t))
    return x


def denoise(W: Dict[str, np.ndarray], cfg, noise: np.ndarray, state: np.ndarray,
            prefix_kv: np.ndarray, n_steps: int) -> np.ndarray:
    """Action chunks [B][H][A] from noise [B][H][A], state [B][Sd] and the
    prefix cache [L][2][B][P][Hkv][D]; each batch element is independent."""
    out = []
    for b in range(noise.shape[0]):
        pk, pv = prefix_kv[:, 0, b], prefix_kv[:, 1, b]
        vel = (lambda x, t, b=b, pk=pk, pv=pv:
               expert_velocity(W, cfg, x, state[b], t, pk, pv))
        out.append(euler_integrate(vel, noise[b], n_steps))
    return np.stack(out)


# ---------------------------------------------------------------------------
# FLASH parallel verification
# ---------------------------------------------------------------------------

def interpolate(draft: np.ndarray, eps: np.ndarray, tau: float) -> np.ndarray:
    """X_tau = tau * eps + (1 - tau) * D   ([DM0.5] 5.3 path, [FLASH] 02)."""
    return F64(tau) * eps + (1.0 - F64(tau)) * draft


def endpoint(x_tau: np.ndarray, tau: float, v: np.ndarray) -> np.ndarray:
    """Rebuilt endpoint A_hat = X_tau - tau * v   ([FLASH] 02)."""
    return x_tau - F64(tau) * v


def gripper_switch_rows(draft: np.ndarray, gripper_dim: int) -> np.ndarray:
    """Rows h in [1, H) where the gripper's sign (value > 0) differs from row h-1."""
    s = np.asarray(draft)[:, gripper_dim] > 0
    return np.nonzero(s[1:] != s[:-1])[0] + 1


def verify_decide(dist: np.ndarray, draft: np.ndarray, delta: float,
                  gripper_dim: int) -> Tuple[int, int]:
    """Accepted length and flags from the distances d[T][H] ([FLASH] 03.2-03.3, reading R9).

    The comparison d < delta is taken in float32, the precision in which the
    device computes d.
    """
    passed = np.all(np.asarray(dist, dtype=np.float32) < np.float32(delta), axis=0)
    n_acc = 0
    while n_acc < passed.shape[0] and passed[n_acc]:
        n_acc += 1
    sw = gripper_switch_rows(draft, gripper_dim)
    flags = 0
    if n_acc == 0:
        flags |= FLAG_ZERO_ACCEPT
    if sw.size:
        flags |= FLAG_SWITCH
    if np.any(sw < n_acc):
        flags |= FLAG_SWITCH_IN_PREFIX
    return n_acc, flags


def fallback(flags: int) -> bool:
    """Full path is taken on zero accepted length or a gripper switch ([FLASH] 03.2-03.3)."""
    return bool(flags & (FLAG_ZERO_ACCEPT | FLAG_SWITCH))


def verify_with_velocity(velocity: Callable[[np.ndarray, float], np.ndarray], draft: np.ndarray,
                         eps: np.ndarray, taus: Sequence[float], delta: float,
                         gripper_dim: int) -> Tuple[int, int, np.ndarray]:
    """Interpolate, predict, rebuild and compare at every tau ([FLASH] 02, 03.2).

    Returns (accepted length, flags, d[T][H]).
    """
    draft = np.asarray(draft, dtype=F64)
    eps = np.asarray(eps, dtype=F64)
    dist = np.zeros((len(taus), draft.shape[0]), dtype=F64)
    for i, tau in enumerate(taus):
        x_tau = interpolate(draft, eps, tau)
        a_hat = endpoint(x_tau, tau, velocity(x_tau, float(tau)))
        dist[i] = np.sqrt(np.sum((a_hat - draft) ** 2, axis=1))
    n_acc, flags = verify_decide(dist, draft, delta, gripper_dim)
    return n_acc, flags, dist


def verify(W: Dict[str, np.ndarray], cfg, draft: np.ndarray, eps: np.ndarray, state: np.ndarray,
           prefix_kv: np.ndarray, taus: Sequence[float], delta: float,
           gripper_dim: int) -> Tuple[int, int, np.ndarray]:
    """FLASH verification of one draft chunk with the action expert.

    draft, eps [H][A]; state [Sd]; prefix_kv [L][2][1][P][Hkv][D].  Every tau
    sees the shared prefix and its own suffix only.
    """
    pk, pv = prefix_kv[:, 0, 0], prefix_kv[:, 1, 0]
    vel = lambda x, t: expert_velocity(W, cfg, x, state, t, pk, pv)  # noqa: E731
    return verify_with_velocity(vel, draft, eps, taus, delta, gripper_dim)
