"""Plain CPU oracle of the GPT-2 (124M) training step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module: only
tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference arm may.
It shares no code with the CUDA library; the only common module is the seeded input
generator (decoder_only_transformer_train_b200.synthetic), which holds none of the
method's arithmetic.

Every step is the plain definition, written with torch CPU tensor ops in the dtype
of the inputs (float64 for parity checks, float32 for the timed CPU baseline).
Matrix products use torch.matmul as a library primitive; nothing is blocked, fused
or reordered.  The backward pass is the analytic gradient of each op, written out
(no autograd); tests pin it to finite differences and to an independent autograd
formulation.

Citations name a page and a section on it:
  [L9]  "Karpathy's Zero to Hero, Lecture 9: Reproduce GPT-2 (124M) — notes, code and
        timestamps" (longvideonotes.com)
  [RG2] "reproduce-gpt2" README (github zzkai098/reproduce-gpt2)
Readings where the pages are silent (LayerNorm eps, AdamW details, clip formula,
argmax ties, ignore index) are marked READING.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

IGNORE_INDEX = -1


@dataclass(frozen=True)
class Config:
    """[L9] "13:34 – 28:07 Writing GPT-2 as a PyTorch module" (GPTConfig) and
    "2:06:39 – 2:14:58 Nice numbers: padding the vocabulary" (padded_vocab_size)."""
    n_layer: int = 12
    n_embd: int = 768
    n_head: int = 12
    block_size: int = 1024
    vocab_size: int = 50257          # real vocabulary: ids and targets live in [0, vocab_size)
    padded_vocab_size: int = 50304   # rows of wte and columns of the logits

    @property
    def head_dim(self) -> int:
        return self.n_embd // self.n_head


GPT2_124M = Config()
TINY = Config(n_layer=2, n_embd=64, n_head=4, block_size=64, vocab_size=512, padded_vocab_size=512)

LAYER_PARAMS = ("ln_1.weight", "ln_1.bias", "attn.c_attn.weight", "attn.c_attn.bias",
                "attn.c_proj.weight", "attn.c_proj.bias", "ln_2.weight", "ln_2.bias",
                "mlp.c_fc.weight", "mlp.c_fc.bias", "mlp.c_proj.weight", "mlp.c_proj.bias")


def param_specs(cfg: Config) -> list[tuple[str, tuple[int, ...]]]:
    """Canonical parameter order and shapes (Hugging Face names, [L9] "Code you'll
    write", model skeleton).  nn.Linear weights are [out, in].  lm_head is wte (tied,
    [L9] "1:06:18 – 1:13:27 Weight tying"), so it is listed once."""
    C, V, T = cfg.n_embd, cfg.padded_vocab_size, cfg.block_size
    specs = [("wte", (V, C)), ("wpe", (T, C))]
    shapes = {"ln_1.weight": (C,), "ln_1.bias": (C,),
              "attn.c_attn.weight": (3 * C, C), "attn.c_attn.bias": (3 * C,),
              "attn.c_proj.weight": (C, C), "attn.c_proj.bias": (C,),
              "ln_2.weight": (C,), "ln_2.bias": (C,),
              "mlp.c_fc.weight": (4 * C, C), "mlp.c_fc.bias": (4 * C,),
              "mlp.c_proj.weight": (C, 4 * C), "mlp.c_proj.bias": (C,)}
    for l in range(cfg.n_layer):
        for p in LAYER_PARAMS:
            specs.append((f"h.{l}.{p}", shapes[p]))
    specs += [("ln_f.weight", (C,)), ("ln_f.bias", (C,))]
    return specs


def is_decayed(name: str, shape: tuple[int, ...]) -> bool:
    """[L9] "2:25:57 – 2:34:49 Batch ramp, weight decay and fused AdamW": tensors with two
    or more dimensions decay, biases and LayerNorm parameters do not."""
    return len(shape) >= 2


def num_params(cfg: Config, vocab_rows: int | None = None) -> int:
    V = cfg.padded_vocab_size if vocab_rows is None else vocab_rows
    total = 0
    for name, shape in param_specs(cfg):
        total += (V * shape[1]) if name == "wte" else int(np.prod(shape))
    return total


# ----------------------------------------------------------------------------- init
# Initialisation per [L9] "1:13:27 – 1:22:16 Matching GPT-2's initialization" and [RG2]
# "Initialization": N(0, 0.02) for Linear and Embedding weights (both embeddings at 0.02),
# zero biases, LayerNorm weight 1 and bias 0, residual projections (attn.c_proj,
# mlp.c_proj) at 0.02 * (2 * n_layer) ** -0.5.  The tied tensor is drawn once.
#
# The pages fix no generator.  Both this oracle and the CUDA library implement the same
# counter-based draw from its published definition (SplitMix64, Steele et al. 2014, with
# the Box–Muller transform):
#   state_t    = SplitMix64 output number t of `seed`  (t = index in param_specs order)
#   r_j        = SplitMix64 output number j of state_t
#   element e  : u1 = 1 - (r_{2e} >> 11) * 2^-53,  u2 = (r_{2e+1} >> 11) * 2^-53
#                z  = sqrt(-2 ln u1) * cos(2 pi u2)   (double), value = float32(std * z)

_G = 0x9E3779B97F4A7C15
_MASK = 0xFFFFFFFFFFFFFFFF


def _splitmix64_outputs(state: int, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = np.uint64(state) + (idx.astype(np.uint64) + np.uint64(1)) * np.uint64(_G)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def _init_std(name: str, cfg: Config) -> float | None:
    if name.endswith(".bias") or name.startswith("ln_f") or ".ln_" in name:
        return None                                     # constant init
    std = 0.02
    if name.endswith("attn.c_proj.weight") or name.endswith("mlp.c_proj.weight"):
        std *= (2 * cfg.n_layer) ** -0.5
    return std


def init_params(cfg: Config, seed: int, dtype=torch.float64) -> dict[str, torch.Tensor]:
    params = {}
    for t, (name, shape) in enumerate(param_specs(cfg)):
        std = _init_std(name, cfg)
        n = int(np.prod(shape))
        if std is None:
            val = np.ones(n) if name.endswith(".weight") else np.zeros(n)
            params[name] = torch.tensor(val, dtype=dtype).reshape(shape)
            continue
        state = int(_splitmix64_outputs(seed & _MASK, np.array([t]))[0])
        r = _splitmix64_outputs(state, np.arange(2 * n, dtype=np.uint64)).reshape(n, 2)
        u1 = 1.0 - (r[:, 0] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        u2 = (r[:, 1] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        vals = (std * z).astype(np.float32)             # the stored parameter is fp32
        params[name] = torch.from_numpy(vals).to(dtype).reshape(shape)
    return params


def flatten(tensors: dict[str, torch.Tensor], cfg: Config) -> torch.Tensor:
    return torch.cat([tensors[n].reshape(-1) for n, _ in param_specs(cfg)])


def unflatten(flat: torch.Tensor, cfg: Config) -> dict[str, torch.Tensor]:
    out, off = {}, 0
    for name, shape in param_specs(cfg):
        n = int(np.prod(shape))
        out[name] = flat[off:off + n].reshape(shape).clone()
        off += n
    assert off == flat.numel()
    return out


# ----------------------------------------------------------------------------- ops
def layernorm_forward(x, w, b, eps=1e-5):
    """nn.LayerNorm(C) over the last dim ([L9] "Code you'll write", Block).
    READING: eps = 1e-5 (module default) and the biased variance (divide by C)."""
    mean = x.mean(dim=-1, keepdim=True)
    var = ((x - mean) ** 2).mean(dim=-1, keepdim=True)
    rstd = 1.0 / torch.sqrt(var + eps)
    y = (x - mean) * rstd * w + b
    return y, mean.squeeze(-1), rstd.squeeze(-1)


def layernorm_backward(dy, x, w, mean, rstd):
    """Analytic gradient of layernorm_forward: returns (dx, dw, db)."""
    xhat = (x - mean.unsqueeze(-1)) * rstd.unsqueeze(-1)
    dxhat = dy * w
    dx = rstd.unsqueeze(-1) * (dxhat - dxhat.mean(dim=-1, keepdim=True)
                               - xhat * (dxhat * xhat).mean(dim=-1, keepdim=True))
    red = tuple(range(dy.dim() - 1))
    return dx, (dy * xhat).sum(dim=red), dy.sum(dim=red)


_GELU_A = math.sqrt(2.0 / math.pi)
_GELU_C = 0.044715


def gelu_tanh(x):
    """The tanh approximation GPT-2 used ([L9] "1:48:25 – 2:00:19 torch.compile and the
    GPU memory hierarchy", the hand-written TanhGELU)."""
    return 0.5 * x * (1.0 + torch.tanh(_GELU_A * (x + _GELU_C * x ** 3)))


def gelu_tanh_grad(x):
    """d gelu_tanh / dx."""
    t = torch.tanh(_GELU_A * (x + _GELU_C * x ** 3))
    return 0.5 * (1.0 + t) + 0.5 * x * (1.0 - t * t) * _GELU_A * (1.0 + 3.0 * _GELU_C * x * x)


def causal_attention_forward(q, k, v):
    """The four-line attention ([L9] "13:34 – 28:07 Writing GPT-2 as a PyTorch module"):
    scores q k^T / sqrt(hd), causal mask (key j > query i gets -inf), softmax over keys,
    weighted sum of values.  q, k, v: [B, H, T, hd].  Returns (o, p) with p [B, H, T, T].
    READING: the scale is SDPA's default 1/sqrt(hd)."""
    T, hd = q.shape[-2], q.shape[-1]
    s = torch.matmul(q, k.transpose(-1, -2)) * (1.0 / math.sqrt(hd))
    mask = torch.ones(T, T, dtype=torch.bool).triu(1)
    s = s.masked_fill(mask, float("-inf"))
    s = s - s.max(dim=-1, keepdim=True).values
    e = torch.exp(s)
    p = e / e.sum(dim=-1, keepdim=True)
    return torch.matmul(p, v), p


def causal_attention_backward(do, q, k, v, p):
    """Gradient of causal_attention_forward given its probabilities p."""
    hd = q.shape[-1]
    scale = 1.0 / math.sqrt(hd)
    dv = torch.matmul(p.transpose(-1, -2), do)
    dp = torch.matmul(do, v.transpose(-1, -2))
    ds = p * (dp - (dp * p).sum(dim=-1, keepdim=True))     # softmax Jacobian-vector product
    dq = torch.matmul(ds, k) * scale
    dk = torch.matmul(ds.transpose(-1, -2), q) * scale
    return dq, dk, dv


def cross_entropy_forward(logits, targets):
    """F.cross_entropy on flattened logits ([L9] "52:38 – 1:06:18 Loss, AdamW and a tiny
    data loader"): mean over rows of logsumexp(z) - z[y].  All padded_vocab_size columns
    are in the normaliser ([L9] "2:06:39 – 2:14:58": pad rows become extra output logits).
    READING: rows whose target is IGNORE_INDEX are left out of the mean.
    Returns (loss, lse [N], valid-count)."""
    m = logits.max(dim=-1, keepdim=True).values
    lse = (m + torch.log(torch.exp(logits - m).sum(dim=-1, keepdim=True))).squeeze(-1)
    valid = targets != IGNORE_INDEX
    count = int(valid.sum())
    tz = logits.gather(1, targets.clamp(min=0).unsqueeze(1)).squeeze(1)
    per_row = torch.where(valid, lse - tz, torch.zeros_like(lse))
    loss = per_row.sum() / max(count, 1)
    return loss, lse, count


def cross_entropy_backward(logits, targets, lse, count, grad_scale):
    """d(grad_scale * loss)/d logits = grad_scale * (softmax(z) - onehot(y)) / count,
    zero on ignored rows."""
    p = torch.exp(logits - lse.unsqueeze(1))
    valid = targets != IGNORE_INDEX
    rows = torch.nonzero(valid).squeeze(1)
    p[rows, targets[rows].long()] -= 1.0
    p[~valid] = 0.0
    return p * (grad_scale / max(count, 1))


def argmax_lowest(logits):
    """READING: argmax over all padded_vocab_size columns, ties to the lowest index."""
    m = logits.max(dim=-1, keepdim=True).values
    idx = torch.arange(logits.shape[-1]).expand_as(logits)
    return torch.where(logits == m, idx, logits.shape[-1]).min(dim=-1).values.to(torch.int32)


def sample_top_k(logits_row, k: int, u: float):
    """Next-token sampling from one row of logits ([L9] "28:07 – 41:44 Loading the weights
    and generating text": softmax, keep the 50 most probable tokens, renormalise, draw one;
    "3:22:33 – 3:28:16 Validation loss and sampling during training": the draw uses its own
    seeded generator).  READINGS: the kept tokens are the k largest logits, ties to the
    lower index, in descending order (the top-k of the softmax is the top-k of the logits);
    the draw is the inverse CDF of the renormalised probabilities in that order at the
    uniform u in [0, 1): the first j whose cumulative probability exceeds u.
    Returns (token, kept token ids in order)."""
    z = [float(v) for v in logits_row]
    k = min(k, len(z))
    order = sorted(range(len(z)), key=lambda i: (-z[i], i))[:k]
    w = [math.exp(z[i] - z[order[0]]) for i in order]
    total = math.fsum(w)
    target = u * total
    cum = 0.0
    for j, wj in enumerate(w):
        cum += wj
        if cum > target:
            return order[j], order
    return order[-1], order


# ----------------------------------------------------------------------------- model
def encoder_forward(wte, wpe, tokens):
    """x0[b, t] = wte[tokens[b, t]] + wpe[t] ([L9] "Code you'll write", forward pass:
    token embedding plus position embedding).  tokens: int [B, T]."""
    tok = torch.as_tensor(tokens).long()
    return wte[tok] + wpe[: tok.shape[1]].unsqueeze(0)


def forward(params, cfg: Config, tokens, targets=None):
    """GPT.forward ([L9] "Code you'll write", forward pass with loss): token + position
    embedding, n_layer pre-LayerNorm blocks x = x + attn(ln_1(x)); x = x + mlp(ln_2(x)),
    ln_f, tied lm_head, cross-entropy.  tokens/targets: int [B, T].
    Returns (loss or None, cache)."""
    B, T = tokens.shape
    assert T <= cfg.block_size
    C, H, hd = cfg.n_embd, cfg.n_head, cfg.head_dim
    tok = torch.as_tensor(tokens).long()
    x = encoder_forward(params["wte"], params["wpe"], tok)            # [B, T, C]
    cache = {"tokens": tok, "layers": [], "B": B, "T": T}
    for l in range(cfg.n_layer):
        P = lambda n: params[f"h.{l}.{n}"]
        lc = {"x": x}
        y1, m1, r1 = layernorm_forward(x, P("ln_1.weight"), P("ln_1.bias"))
        qkv = torch.matmul(y1, P("attn.c_attn.weight").T) + P("attn.c_attn.bias")
        q, k, v = qkv.split(C, dim=-1)
        heads = lambda t: t.reshape(B, T, H, hd).transpose(1, 2)       # [B, H, T, hd]
        o, _ = causal_attention_forward(heads(q), heads(k), heads(v))
        o = o.transpose(1, 2).reshape(B, T, C)
        x1 = x + torch.matmul(o, P("attn.c_proj.weight").T) + P("attn.c_proj.bias")
        y2, m2, r2 = layernorm_forward(x1, P("ln_2.weight"), P("ln_2.bias"))
        u = torch.matmul(y2, P("mlp.c_fc.weight").T) + P("mlp.c_fc.bias")
        g = gelu_tanh(u)
        x = x1 + torch.matmul(g, P("mlp.c_proj.weight").T) + P("mlp.c_proj.bias")
        lc.update(y1=y1, m1=m1, r1=r1, qkv=qkv, o=o, x1=x1, y2=y2, m2=m2, r2=r2, u=u, g=g)
        cache["layers"].append(lc)
    h, mf, rf = layernorm_forward(x, params["ln_f.weight"], params["ln_f.bias"])
    logits = torch.matmul(h, params["wte"].T).reshape(B * T, -1)     # [N, Vp]
    cache.update(xL=x, h=h, mf=mf, rf=rf, logits=logits)
    if targets is None:
        return None, cache
    tg = torch.as_tensor(targets).reshape(-1).long()
    loss, lse, count = cross_entropy_forward(logits, tg)
    cache.update(targets=tg, lse=lse, count=count)
    return loss, cache


def backward(params, cfg: Config, cache, grad_scale: float = 1.0, grads=None):
    """Gradients of grad_scale * loss, added into `grads` (a dict like params, created
    zero if None).  With grad_scale = 1/k over k micro-steps this is the accumulation of
    [L9] "2:34:49 – 2:46:43 Gradient accumulation" (loss divided by the micro-step count,
    gradients summed).  The tied wte receives the lm_head and the embedding gradients
    ([L9] "1:06:18 – 1:13:27 Weight tying")."""
    if grads is None:
        grads = {n: torch.zeros_like(t) for n, t in params.items()}
    B, T = cache["B"], cache["T"]
    C, H, hd = cfg.n_embd, cfg.n_head, cfg.head_dim
    dz = cross_entropy_backward(cache["logits"], cache["targets"], cache["lse"],
                                cache["count"], grad_scale)               # [N, Vp]
    h = cache["h"].reshape(B * T, C)
    grads["wte"] += torch.matmul(dz.T, h)
    dh = torch.matmul(dz, params["wte"]).reshape(B, T, C)
    dx, dwf, dbf = layernorm_backward(dh, cache["xL"], params["ln_f.weight"], cache["mf"], cache["rf"])
    grads["ln_f.weight"] += dwf
    grads["ln_f.bias"] += dbf
    heads = lambda t: t.reshape(B, T, H, hd).transpose(1, 2)
    for l in reversed(range(cfg.n_layer)):
        P = lambda n: params[f"h.{l}.{n}"]
        lc = cache["layers"][l]
        G = lambda n, val: grads[f"h.{l}.{n}"].__iadd__(val)
        flat = lambda t: t.reshape(B * T, -1)
        # x_out = x1 + g W_mp^T + b_mp
        G("mlp.c_proj.weight", flat(dx).T @ flat(lc["g"]))
        G("mlp.c_proj.bias", flat(dx).sum(0))
        dg = torch.matmul(dx, P("mlp.c_proj.weight"))
        du = dg * gelu_tanh_grad(lc["u"])
        G("mlp.c_fc.weight", flat(du).T @ flat(lc["y2"]))
        G("mlp.c_fc.bias", flat(du).sum(0))
        dy2 = torch.matmul(du, P("mlp.c_fc.weight"))
        dln, dw2, db2 = layernorm_backward(dy2, lc["x1"], P("ln_2.weight"), lc["m2"], lc["r2"])
        G("ln_2.weight", dw2)
        G("ln_2.bias", db2)
        dx1 = dx + dln
        # x1 = x + o W_p^T + b_p
        G("attn.c_proj.weight", flat(dx1).T @ flat(lc["o"]))
        G("attn.c_proj.bias", flat(dx1).sum(0))
        do = torch.matmul(dx1, P("attn.c_proj.weight"))
        q, k, v = lc["qkv"].split(C, dim=-1)
        _, p = causal_attention_forward(heads(q), heads(k), heads(v))   # recomputed
        dq, dk, dv = causal_attention_backward(heads(do), heads(q), heads(k), heads(v), p)
        merge = lambda t: t.transpose(1, 2).reshape(B, T, C)
        dqkv = torch.cat([merge(dq), merge(dk), merge(dv)], dim=-1)
        G("attn.c_attn.weight", flat(dqkv).T @ flat(lc["y1"]))
        G("attn.c_attn.bias", flat(dqkv).sum(0))
        dy1 = torch.matmul(dqkv, P("attn.c_attn.weight"))
        dln, dw1, db1 = layernorm_backward(dy1, lc["x"], P("ln_1.weight"), lc["m1"], lc["r1"])
        G("ln_1.weight", dw1)
        G("ln_1.bias", db1)
        dx = dx1 + dln
    encoder_backward(grads, cache["tokens"], dx)
    return grads


def encoder_backward(grads, tokens, dx0):
    """x0 = wte[tok] + wpe[t]: dwte[v] += sum of dx0 over positions holding token v;
    dwpe[t] += sum over the batch of dx0[:, t]."""
    B, T, C = dx0.shape
    grads["wte"].index_add_(0, tokens.reshape(-1), dx0.reshape(B * T, C))
    grads["wpe"][:T] += dx0.sum(dim=0)


# ----------------------------------------------------------------------------- optimizer
def global_norm(grads, cfg: Config) -> float:
    """sqrt of the sum of squares of every gradient element; the tied tensor counts once
    ([L9] "2:14:58 – 2:25:57 GPT-3's optimizer recipe", gradient clipping)."""
    return math.sqrt(sum(float((grads[n].double() ** 2).sum()) for n, _ in param_specs(cfg)))


def clip_scale(norm: float, clip: float) -> float:
    """READING (clip_grad_norm_ semantics): s = min(1, clip / (norm + 1e-6))."""
    return min(1.0, clip / (norm + 1e-6))


def adamw_update(p, g, m, v, t, lr, beta1, beta2, eps, wd):
    """Decoupled weight decay AdamW (Loshchilov & Hutter) with Adam's bias correction
    (Kingma & Ba), as torch.optim.AdamW: [L9] "2:14:58 – 2:25:57" (betas 0.9/0.95, eps
    1e-8) and "2:25:57 – 2:34:49" (weight decay 0.1 on >=2-D tensors).
    READING: decay p *= 1 - lr*wd first, then the moment update, eps added after the
    square root of the bias-corrected second moment, t counted from 1.  Returns new
    (p, m, v)."""
    p = p * (1.0 - lr * wd)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    return p - lr * mhat / (torch.sqrt(vhat) + eps), m, v


def optimizer_step(params, grads, m, v, t, cfg: Config, lr, beta1=0.9, beta2=0.95, eps=1e-8,
                   wd=0.1, clip=1.0):
    """Clip by global norm, then AdamW on every tensor (wd only where is_decayed).
    Updates params, m, v in place; returns the pre-clip norm."""
    norm = global_norm(grads, cfg)
    s = clip_scale(norm, clip)
    for name, shape in param_specs(cfg):
        w = wd if is_decayed(name, shape) else 0.0
        params[name], m[name], v[name] = adamw_update(
            params[name], grads[name] * s, m[name], v[name], t, lr, beta1, beta2, eps, w)
    return norm


def get_lr(it: int, max_lr=6e-4, warmup_steps=715, max_steps=19073, min_ratio=0.1) -> float:
    """[L9] "2:14:58 – 2:25:57 GPT-3's optimizer recipe" and "Code you'll write": linear
    warmup (it+1)/warmup * max_lr, then cosine decay to min_ratio * max_lr at max_steps,
    constant afterwards."""
    min_lr = max_lr * min_ratio
    if it < warmup_steps:
        return max_lr * (it + 1) / warmup_steps
    if it > max_steps:
        return min_lr
    ratio = (it - warmup_steps) / (max_steps - warmup_steps)
    return min_lr + 0.5 * (1.0 + math.cos(math.pi * ratio)) * (max_lr - min_lr)


def train_step(params, m, v, t, cfg: Config, batches, lr, **opt):
    """One optimizer step over k = len(batches) micro-batches (loss/k per micro-step):
    zero_grad, k x (forward, backward), clip, AdamW.  Returns (mean loss, norm, grads)."""
    k = len(batches)
    grads = {n: torch.zeros_like(p) for n, p in params.items()}
    loss_accum = 0.0
    for tokens, targets in batches:
        loss, cache = forward(params, cfg, tokens, targets)
        backward(params, cfg, cache, grad_scale=1.0 / k, grads=grads)
        loss_accum += float(loss) / k
    norm = optimizer_step(params, grads, m, v, t, cfg, lr, **opt)
    return loss_accum, norm, grads
