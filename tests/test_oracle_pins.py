"""Pins of the CPU oracle to things other than itself: figures printed on the pages,
closed forms, invariants, brute force, finite differences, and library routines
(torch autograd, torch.optim.AdamW, clip_grad_norm_) that compute the same definitions.

Each test is chosen so that a plausible mistake in the oracle (a dropped term, a wrong
sign, a transposed operand, a wrong index) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from decoder_only_transformer_train_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PAGES = json.load(open(os.path.join(GOLDEN, "pages_figures.json")))
D = torch.float64

# a small config that still has several heads, layers and a padded vocabulary
SMALL = O.Config(n_layer=2, n_embd=32, n_head=4, block_size=16, vocab_size=97, padded_vocab_size=104)


def _batch(cfg, seed=2, B=2, T=None, step=0):
    T = T or cfg.block_size
    x, y = S.token_batch(seed, B, T, cfg.vocab_size, micro_step=step)
    return torch.from_numpy(x), torch.from_numpy(y)


def _perturbed_params(cfg, seed=1):
    """Init, then move biases / LN params off their constants so every term is live."""
    p = O.init_params(cfg, seed, dtype=D)
    g = torch.Generator().manual_seed(seed)
    for n, t in p.items():
        if t.dim() == 1:
            p[n] = t + 0.1 * torch.randn(t.shape, generator=g, dtype=D)
    return p


# ----------------------------------------------------------------- figures on the pages
def test_param_counts_match_pages():
    cfg = O.GPT2_124M
    assert O.num_params(cfg, vocab_rows=50257) == PAGES["param_count_vocab_50257"]["value"]
    specs = O.param_specs(cfg)
    dec = [(n, s) for n, s in specs if O.is_decayed(n, s)]
    nod = [(n, s) for n, s in specs if not O.is_decayed(n, s)]
    assert len(dec) == PAGES["decayed_tensors"]["value"]
    assert len(nod) == PAGES["nondecayed_tensors"]["value"]
    assert sum(int(np.prod(s)) for _, s in dec) == PAGES["decayed_params"]["value"]
    assert sum(int(np.prod(s)) for _, s in nod) == PAGES["nondecayed_params"]["value"]
    shapes = dict(specs)
    assert list(shapes["wpe"]) == PAGES["wpe_shape"]["value"]
    assert shapes["wte"][1] == PAGES["wte_shape_hf"]["value"][1]
    assert cfg.padded_vocab_size == PAGES["padded_vocab"]["value"]
    assert O.num_params(O.TINY) == 136960


def test_lr_schedule_matches_page_constants():
    g = lambda k: PAGES[k]["value"]
    kw = dict(max_lr=g("lr_max"), warmup_steps=g("warmup_steps"), max_steps=g("max_steps"),
              min_ratio=g("lr_min_ratio"))
    assert O.get_lr(0, **kw) == pytest.approx(6e-4 / 715, rel=1e-12)
    assert O.get_lr(714, **kw) == pytest.approx(6e-4, rel=1e-12)
    assert O.get_lr(715, **kw) == pytest.approx(6e-4, rel=1e-12)       # cosine starts at the peak
    assert O.get_lr(19073, **kw) == pytest.approx(6e-5, rel=1e-12)     # fully decayed
    assert O.get_lr(30000, **kw) == pytest.approx(6e-5, rel=1e-12)
    mid = (715 + 19073) / 2
    assert O.get_lr(int(mid), **kw) == pytest.approx(6e-5 + 0.5 * 5.4e-4, rel=1e-3)
    assert O.get_lr(1000, **kw) == pytest.approx(5.9967894e-4, rel=1e-7)
    lrs = [O.get_lr(i, **kw) for i in range(715, 19074, 97)]
    assert all(a >= b for a, b in zip(lrs, lrs[1:]))                    # monotone decay


def test_initial_loss_near_uniform_tiny():
    cfg = O.TINY
    p = O.init_params(cfg, 1, dtype=D)
    x, y = _batch(cfg)
    loss, _ = O.forward(p, cfg, x, y)
    assert abs(float(loss) - math.log(cfg.padded_vocab_size)) < 0.1


@pytest.mark.slow
def test_initial_loss_near_uniform_124m():
    cfg = O.GPT2_124M
    p = O.init_params(cfg, 1, dtype=torch.float32)
    x, y = S.token_batch(2, 1, 128, cfg.vocab_size)
    loss, _ = O.forward(p, cfg, torch.from_numpy(x), torch.from_numpy(y))
    # the pages: -ln(1/50257) ~ 10.82 expected, 11.0886 observed at init
    assert abs(float(loss) - PAGES["initial_loss_uniform"]["value"]) < 0.5
    assert abs(float(loss) - PAGES["initial_loss_observed"]["value"]) < 0.5


# ----------------------------------------------------------------- generators
def test_splitmix64_published_vectors():
    gv = json.load(open(os.path.join(GOLDEN, "splitmix64_vectors.json")))
    out = O.gpt2_oracle._splitmix64_outputs(gv["seed"], np.arange(5))
    assert [int(v) for v in out] == [int(s) for s in gv["outputs"]]
    out2 = S.splitmix64(gv["seed"], np.arange(5))
    assert [int(v) for v in out2] == [int(s) for s in gv["outputs"]]


def test_init_scheme_statistics():
    cfg = O.Config(n_layer=4, n_embd=128, n_head=4, block_size=64, vocab_size=1000, padded_vocab_size=1024)
    p = O.init_params(cfg, 7, dtype=D)
    for name, t in p.items():
        if name.endswith(".bias") or ".ln_" in name or name.startswith("ln_f"):
            want = 1.0 if name.endswith(".weight") else 0.0
            assert torch.all(t == want), name
            continue
        std = 0.02 * ((2 * cfg.n_layer) ** -0.5 if name.endswith("c_proj.weight") else 1.0)
        n = t.numel()
        assert abs(float(t.mean())) < 5 * std / math.sqrt(n), name
        assert float(t.std()) == pytest.approx(std, rel=6 / math.sqrt(n) + 0.01), name
    # distinct tensors get distinct draws; the draw is a pure function of (seed, tensor, index)
    assert not torch.equal(p["h.0.attn.c_attn.weight"][:8], p["h.1.attn.c_attn.weight"][:8])
    p2 = O.init_params(cfg, 7, dtype=D)
    assert all(torch.equal(p[n], p2[n]) for n in p)


def test_zipf_stream_shape_and_law():
    x, y = S.token_batch(3, 4, 256, 50257)
    assert x.shape == (4, 256) and x.dtype == np.int32
    assert np.array_equal(x.reshape(-1)[1:], y.reshape(-1)[:-1])     # targets are inputs shifted by one
    ids = S.zipf_tokens(3, 200000, 50257)
    assert ids.min() >= 0 and ids.max() < 50257
    w = np.arange(1, 50258, dtype=np.float64) ** -1.1
    p0 = w[0] / w.sum()
    assert np.mean(ids == 0) == pytest.approx(p0, rel=0.03)
    assert np.mean(ids == 1) == pytest.approx(w[1] / w.sum(), rel=0.05)


# ----------------------------------------------------------------- elementary ops
def test_layernorm_against_library_and_invariants():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(7, 48, generator=g, dtype=D) * 3 + 1
    w = torch.randn(48, generator=g, dtype=D)
    b = torch.randn(48, generator=g, dtype=D)
    y, mean, rstd = O.layernorm_forward(x, w, b)
    assert torch.allclose(y, F.layer_norm(x, (48,), w, b, eps=1e-5), atol=1e-12)
    y0, _, _ = O.layernorm_forward(x, torch.ones(48, dtype=D), torch.zeros(48, dtype=D))
    var = x.var(dim=-1, unbiased=False)
    assert torch.allclose(y0.mean(-1), torch.zeros(7, dtype=D), atol=1e-12)
    assert torch.allclose((y0 ** 2).mean(-1), var / (var + 1e-5), atol=1e-12)
    dy = torch.randn(7, 48, generator=g, dtype=D)
    dx, dw, db = O.layernorm_backward(dy, x, w, mean, rstd)
    xr, wr, br = (t.clone().requires_grad_() for t in (x, w, b))
    F.layer_norm(xr, (48,), wr, br, eps=1e-5).backward(dy)
    for a, r in ((dx, xr.grad), (dw, wr.grad), (db, br.grad)):
        assert torch.allclose(a, r, atol=1e-11)
    assert torch.allclose(dx.sum(-1), torch.zeros(7, dtype=D), atol=1e-11)  # dx orthogonal to 1


def test_gelu_against_library_and_derivative():
    x = torch.linspace(-8, 8, 2001, dtype=D)
    assert torch.allclose(O.gelu_tanh(x), F.gelu(x, approximate="tanh"), atol=1e-14)
    h = 1e-6
    fd = (O.gelu_tanh(x + h) - O.gelu_tanh(x - h)) / (2 * h)
    assert torch.allclose(O.gelu_tanh_grad(x), fd, atol=1e-8)
    assert float(O.gelu_tanh(torch.tensor(0.0, dtype=D))) == 0.0
    assert float(O.gelu_tanh_grad(torch.tensor(0.0, dtype=D))) == 0.5


def _brute_force_attention(q, k, v):
    """Pure-Python loops: o_i = sum_{j<=i} softmax_j(q_i.k_j / sqrt(hd)) v_j."""
    T, hd = len(q), len(q[0])
    out = []
    for i in range(T):
        s = [sum(q[i][d] * k[j][d] for d in range(hd)) / math.sqrt(hd) for j in range(i + 1)]
        m = max(s)
        e = [math.exp(a - m) for a in s]
        z = sum(e)
        out.append([sum(e[j] / z * v[j][d] for j in range(i + 1)) for d in range(hd)])
    return out


def test_attention_brute_force_and_degenerate_cases():
    g = torch.Generator().manual_seed(1)
    q, k, v = (torch.randn(1, 2, 9, 5, generator=g, dtype=D) for _ in range(3))
    o, p = O.causal_attention_forward(q, k, v)
    for h in range(2):
        ref = _brute_force_attention(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist())
        assert torch.allclose(o[0, h], torch.tensor(ref, dtype=D), atol=1e-13)
    assert torch.all(p.triu(1) == 0)
    assert torch.allclose(p.sum(-1), torch.ones(1, 2, 9, dtype=D), atol=1e-14)
    # T = 1: the output is exactly v
    o1, _ = O.causal_attention_forward(q[..., :1, :], k[..., :1, :], v[..., :1, :])
    assert torch.equal(o1, v[..., :1, :])
    # first query always sees only the first key
    assert torch.allclose(o[..., 0, :], v[..., 0, :], atol=0)
    # backward against autograd of an independent expression
    qr, kr, vr = (t.clone().requires_grad_() for t in (q, k, v))
    ref = F.scaled_dot_product_attention(qr, kr, vr, is_causal=True)
    do = torch.randn_like(ref)
    ref.backward(do)
    assert torch.allclose(ref, o, atol=1e-13)
    dq, dk, dv = O.causal_attention_backward(do, q, k, v, p)
    for a, r in ((dq, qr.grad), (dk, kr.grad), (dv, vr.grad)):
        assert torch.allclose(a, r, atol=1e-12)


def test_cross_entropy_library_and_invariants():
    g = torch.Generator().manual_seed(2)
    z = torch.randn(11, 37, generator=g, dtype=D) * 4
    y = torch.randint(0, 30, (11,), generator=g)
    y[3] = O.IGNORE_INDEX
    loss, lse, count = O.cross_entropy_forward(z, y)
    assert count == 10
    assert float(loss) == pytest.approx(float(F.cross_entropy(z, y, ignore_index=-1)), rel=1e-13)
    assert torch.allclose(lse, torch.logsumexp(z, dim=-1), atol=1e-13)
    dz = O.cross_entropy_backward(z, y, lse, count, grad_scale=0.5)
    assert torch.allclose(dz.sum(-1), torch.zeros(11, dtype=D), atol=1e-14)   # rows sum to zero
    assert torch.all(dz[3] == 0)
    p = torch.softmax(z, -1)
    for r in (0, 5, 10):
        assert float(dz[r, y[r]]) == pytest.approx(0.5 * (float(p[r, y[r]]) - 1) / 10, rel=1e-12)
    zr = z.clone().requires_grad_()
    (0.5 * F.cross_entropy(zr, y, ignore_index=-1)).backward()
    assert torch.allclose(dz, zr.grad, atol=1e-14)


def test_argmax_ties_to_lowest_index():
    z = torch.tensor([[1.0, 3.0, 3.0, 0.0], [5.0, 5.0, 5.0, 5.0], [-1.0, -2.0, -3.0, -0.5]], dtype=D)
    assert O.argmax_lowest(z).tolist() == [1, 0, 3]


# ----------------------------------------------------------------- the model
class _AutogradGPT:
    """An independent formulation of the same network through torch.nn.functional and
    autograd, in the pages' style (embedding gather, F.layer_norm, SDPA with is_causal,
    F.gelu tanh, tied lm_head, F.cross_entropy).  Used only to pin the oracle's analytic
    backward."""

    def __init__(self, cfg, params):
        self.cfg = cfg
        self.p = {n: t.clone().requires_grad_() for n, t in params.items()}

    def loss(self, tokens, targets):
        cfg, p = self.cfg, self.p
        B, T = tokens.shape
        C, H = cfg.n_embd, cfg.n_head
        x = F.embedding(tokens.long(), p["wte"]) + F.embedding(torch.arange(T), p["wpe"])
        for l in range(cfg.n_layer):
            q_ = lambda n: p[f"h.{l}.{n}"]
            a = F.layer_norm(x, (C,), q_("ln_1.weight"), q_("ln_1.bias"))
            qkv = F.linear(a, q_("attn.c_attn.weight"), q_("attn.c_attn.bias"))
            qh, kh, vh = (t.view(B, T, H, C // H).transpose(1, 2) for t in qkv.split(C, dim=2))
            att = F.scaled_dot_product_attention(qh, kh, vh, is_causal=True)
            x = x + F.linear(att.transpose(1, 2).reshape(B, T, C), q_("attn.c_proj.weight"), q_("attn.c_proj.bias"))
            m = F.layer_norm(x, (C,), q_("ln_2.weight"), q_("ln_2.bias"))
            m = F.gelu(F.linear(m, q_("mlp.c_fc.weight"), q_("mlp.c_fc.bias")), approximate="tanh")
            x = x + F.linear(m, q_("mlp.c_proj.weight"), q_("mlp.c_proj.bias"))
        x = F.layer_norm(x, (C,), p["ln_f.weight"], p["ln_f.bias"])
        logits = F.linear(x, p["wte"])
        return F.cross_entropy(logits.view(B * T, -1), targets.reshape(-1).long(), ignore_index=-1)


def test_forward_backward_against_autograd_formulation():
    cfg = SMALL
    p = _perturbed_params(cfg)
    x, y = _batch(cfg)
    y[0, 3] = O.IGNORE_INDEX
    loss, cache = O.forward(p, cfg, x, y)
    grads = O.backward(p, cfg, cache, grad_scale=0.25)
    ag = _AutogradGPT(cfg, p)
    ref = ag.loss(x, y)
    (0.25 * ref).backward()
    assert float(loss) == pytest.approx(float(ref.detach()), rel=1e-12)
    for n in p:
        r = ag.p[n].grad
        err = float((grads[n] - r).norm() / (r.norm() + 1e-300))
        assert err < 1e-10, (n, err)


def test_key_bias_gradient_is_zero_by_softmax_shift_invariance():
    """Adding a vector b to every key adds q.b to all scores of a query; the softmax
    ignores a constant shift, so d loss / d (key bias) = 0 exactly."""
    cfg = SMALL
    p = _perturbed_params(cfg)
    x, y = _batch(cfg)
    _, cache = O.forward(p, cfg, x, y)
    g = O.backward(p, cfg, cache)
    C = cfg.n_embd
    for l in range(cfg.n_layer):
        b = g[f"h.{l}.attn.c_attn.bias"]
        assert float(b[C:2 * C].abs().max()) < 1e-12 * float(b.abs().max())
        assert float(b[:C].abs().max()) > 0 and float(b[2 * C:].abs().max()) > 0


def test_finite_differences_every_tensor():
    cfg = SMALL
    p = _perturbed_params(cfg, seed=3)
    x, y = _batch(cfg, seed=4, T=8)
    _, cache = O.forward(p, cfg, x, y)
    grads = O.backward(p, cfg, cache)
    g = torch.Generator().manual_seed(5)
    h = 1e-5
    for name, t in p.items():
        for _ in range(3):
            flat_i = int(torch.randint(0, t.numel(), (1,), generator=g))
            if name == "wpe" and flat_i // cfg.n_embd >= 8:           # rows past T get no gradient
                flat_i %= 8 * cfg.n_embd
            orig = float(t.view(-1)[flat_i])
            t.view(-1)[flat_i] = orig + h
            lp = float(O.forward(p, cfg, x, y)[0])
            t.view(-1)[flat_i] = orig - h
            lm = float(O.forward(p, cfg, x, y)[0])
            t.view(-1)[flat_i] = orig
            fd = (lp - lm) / (2 * h)
            an = float(grads[name].view(-1)[flat_i])
            assert abs(fd - an) <= 1e-4 * max(abs(fd), 1e-3), (name, flat_i, fd, an)


def test_causality_logits_ignore_future_tokens():
    cfg = SMALL
    p = _perturbed_params(cfg)
    x, _ = _batch(cfg, T=16)
    t0 = 9
    x2 = x.clone()
    x2[:, t0 + 1:] = (x2[:, t0 + 1:] * 7 + 3) % cfg.vocab_size
    _, c1 = O.forward(p, cfg, x)
    _, c2 = O.forward(p, cfg, x2)
    l1 = c1["logits"].reshape(2, 16, -1)
    l2 = c2["logits"].reshape(2, 16, -1)
    assert torch.equal(l1[:, : t0 + 1], l2[:, : t0 + 1])
    assert not torch.equal(l1[:, t0 + 1:], l2[:, t0 + 1:])


def test_encoder_backward_invariant():
    cfg = SMALL
    p = _perturbed_params(cfg)
    x, y = _batch(cfg)
    _, cache = O.forward(p, cfg, x, y)
    g = torch.Generator().manual_seed(6)
    dx0 = torch.randn(2, 16, cfg.n_embd, generator=g, dtype=D)
    grads = {n: torch.zeros_like(t) for n, t in p.items()}
    O.encoder_backward(grads, cache["tokens"], dx0)
    tot = dx0.sum(dim=(0, 1))
    assert torch.allclose(grads["wte"].sum(0), tot, atol=1e-12)
    assert torch.allclose(grads["wpe"].sum(0), tot, atol=1e-12)
    v = int(x[0, 0])
    where = (x == v)
    assert torch.allclose(grads["wte"][v], dx0[where].sum(0), atol=1e-12)


def test_encoder_forward_is_adjoint_of_backward():
    """The embedding is linear in (wte, wpe), so <x0, dx0> = <wte, dwte> + <wpe, dwpe>
    for the backward's dwte, dwpe; with wte the identity and wpe zero, x0's rows are the
    one-hot codes of the ids."""
    g = torch.Generator().manual_seed(8)
    V, Tmax, C = 11, 9, 11
    tok = torch.tensor([[3, 3, 0, 10, 7], [1, 3, 9, 9, 2]])
    wte = torch.randn(V, C, generator=g, dtype=D)
    wpe = torch.randn(Tmax, C, generator=g, dtype=D)
    dx0 = torch.randn(2, 5, C, generator=g, dtype=D)
    x0 = O.encoder_forward(wte, wpe, tok)
    grads = {"wte": torch.zeros_like(wte), "wpe": torch.zeros_like(wpe)}
    O.encoder_backward(grads, tok, dx0)
    lhs = float((x0 * dx0).sum())
    rhs = float((wte * grads["wte"]).sum() + (wpe * grads["wpe"]).sum())
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(lhs))
    assert float(grads["wpe"][5:].abs().sum()) == 0.0
    onehot = O.encoder_forward(torch.eye(V, dtype=D), torch.zeros(Tmax, V, dtype=D), tok)
    for b in range(2):
        for t in range(5):
            row = [0.0] * V
            row[int(tok[b, t])] = 1.0
            assert onehot[b, t].tolist() == row


def test_sample_top_k_with_k_one_is_the_argmax():
    g = torch.Generator().manual_seed(31)
    z = torch.randn(3, 40, generator=g, dtype=D)
    z[1, 7] = z[1, 30] = z[1].max() + 1.0          # a tie: the lower index wins
    amax = O.argmax_lowest(z)
    for r in range(3):
        for u in (0.0, 0.37, 0.999999):
            tok, kept = O.sample_top_k(z[r], 1, u)
            assert tok == int(amax[r]) and kept == [tok]
    assert O.sample_top_k(z[1], 1, 0.5)[0] == 7


def test_sample_top_k_frequencies_follow_the_renormalised_softmax():
    """Over a uniform grid of u, each kept token is drawn with the probability
    exp(z_i) / sum over the kept exp(z_j); tokens outside the top k never appear."""
    z = torch.tensor([0.3, 2.0, -1.0, 1.1, 2.0, 0.9, -3.0], dtype=D)
    k = 4
    kept_want = [1, 4, 3, 5]                        # 2.0 (index 1), 2.0 (index 4), 1.1, 0.9
    n = 20000
    counts = {}
    for i in range(n):
        tok, kept = O.sample_top_k(z, k, (i + 0.5) / n)
        assert kept == kept_want
        counts[tok] = counts.get(tok, 0) + 1
    assert set(counts) == set(kept_want)
    e = torch.exp(z[kept_want])
    p = e / e.sum()
    for j, t in enumerate(kept_want):
        assert abs(counts[t] / n - float(p[j])) <= 1.0 / n
    # k >= V keeps every token: the full softmax
    tok_all = [O.sample_top_k(z, 100, (i + 0.5) / n)[0] for i in range(0, n, 10)]
    full = torch.softmax(z, 0)
    for t in range(7):
        assert abs(tok_all.count(t) / len(tok_all) - float(full[t])) <= 10.0 / n + 1e-12


def test_grad_accumulation_equals_one_big_batch():
    """[L9] 2:34:49 – 2:46:43: k micro-steps with loss/k give the full-batch gradient."""
    cfg = SMALL
    p = _perturbed_params(cfg)
    x, y = _batch(cfg, B=4)
    _, cache = O.forward(p, cfg, x, y)
    full = O.backward(p, cfg, cache)
    acc = {n: torch.zeros_like(t) for n, t in p.items()}
    for i in range(4):
        _, c = O.forward(p, cfg, x[i:i + 1], y[i:i + 1])
        O.backward(p, cfg, c, grad_scale=0.25, grads=acc)
    for n in p:
        assert torch.allclose(acc[n], full[n], rtol=1e-10, atol=1e-14), n
    # without the 1/k the gradient is k times too large (the pages' bug)
    wrong = {n: torch.zeros_like(t) for n, t in p.items()}
    for i in range(4):
        _, c = O.forward(p, cfg, x[i:i + 1], y[i:i + 1])
        O.backward(p, cfg, c, grad_scale=1.0, grads=wrong)
    assert torch.allclose(wrong["wte"], 4 * full["wte"], rtol=1e-10, atol=1e-14)


# ----------------------------------------------------------------- optimizer
def test_adamw_first_step_closed_form_and_library():
    g = torch.Generator().manual_seed(8)
    p0 = torch.randn(64, 32, generator=g, dtype=D)
    gr = torch.randn(64, 32, generator=g, dtype=D)
    lr, wd, eps = 6e-4, 0.1, 1e-8
    p1, m1, v1 = O.adamw_update(p0, gr, torch.zeros_like(p0), torch.zeros_like(p0), 1, lr, 0.9, 0.95, eps, wd)
    closed = p0 * (1 - lr * wd) - lr * gr / (gr.abs() + eps)
    assert torch.allclose(p1, closed, rtol=0, atol=1e-15)
    # several steps against torch.optim.AdamW (same definition, library code)
    pr = p0.clone().requires_grad_()
    opt = torch.optim.AdamW([pr], lr=lr, betas=(0.9, 0.95), eps=eps, weight_decay=wd)
    p, m, v = p0.clone(), torch.zeros_like(p0), torch.zeros_like(p0)
    for t in range(1, 6):
        gt = torch.randn(64, 32, generator=g, dtype=D)
        pr.grad = gt.clone()
        opt.step()
        p, m, v = O.adamw_update(p, gt, m, v, t, lr, 0.9, 0.95, eps, wd)
    assert torch.allclose(p, pr.detach(), rtol=0, atol=1e-15)


def test_clip_matches_library_and_closed_form():
    cfg = SMALL
    p = _perturbed_params(cfg)
    x, y = _batch(cfg)
    _, cache = O.forward(p, cfg, x, y)
    grads = O.backward(p, cfg, cache)
    n = O.global_norm(grads, cfg)
    holders = []
    for k, _ in O.param_specs(cfg):
        h = torch.zeros_like(grads[k], requires_grad=True)
        h.grad = grads[k].clone()
        holders.append(h)
    lib = float(torch.nn.utils.clip_grad_norm_(holders, 1.0))
    tensors = [h.grad for h in holders]
    assert n == pytest.approx(lib, rel=1e-12)
    s = O.clip_scale(n, 1.0)
    post = math.sqrt(sum(float(((grads[k] * s) ** 2).sum()) for k, _ in O.param_specs(cfg)))
    if n > 1.0:
        assert post == pytest.approx(n / (n + 1e-6), rel=1e-12)
        assert post == pytest.approx(math.sqrt(sum(float((t ** 2).sum()) for t in tensors)), rel=1e-12)
    assert O.clip_scale(0.5, 1.0) == 1.0


def test_weight_decay_only_on_matrices():
    cfg = SMALL
    p = _perturbed_params(cfg)
    zero = {n: torch.zeros_like(t) for n, t in p.items()}
    m = {n: torch.zeros_like(t) for n, t in p.items()}
    v = {n: torch.zeros_like(t) for n, t in p.items()}
    before = {n: t.clone() for n, t in p.items()}
    O.optimizer_step(p, zero, m, v, 1, cfg, lr=0.5, wd=0.1)
    for name, shape in O.param_specs(cfg):
        if len(shape) >= 2:
            assert torch.allclose(p[name], before[name] * 0.95, atol=1e-15), name
        else:
            assert torch.equal(p[name], before[name]), name


@pytest.mark.slow
def test_overfit_single_batch():
    """[L9] 52:38 – 1:06:18: repeated steps on one batch drive the loss toward zero."""
    cfg = O.Config(n_layer=2, n_embd=64, n_head=4, block_size=32, vocab_size=128, padded_vocab_size=128)
    p = O.init_params(cfg, 1, dtype=torch.float32)
    m = {n: torch.zeros_like(t) for n, t in p.items()}
    v = {n: torch.zeros_like(t) for n, t in p.items()}
    x, y = _batch(cfg, B=2, T=32)
    first = None
    for t in range(1, 81):
        loss, _, _ = O.train_step(p, m, v, t, cfg, [(x, y)], lr=3e-3)
        first = first if first is not None else loss
    assert first > 4.0 and loss < 0.1
