"""Per-operation timing through the single-operation C ABI (gpt2op_*), at the shapes of the
GPT-2 124M training step with B micro-batch rows of T tokens (default B=16, T=1024).

    python -m decoder_only_transformer_train_b200.opbench [--only REGEX] [--iters N]
        [--warmup W] [--flush-l2] [--micro-batch B] [--seq T] [--qkv-std S]

Each case is timed with CUDA events on the current stream over N launches after W warm-up
launches and printed as one line: microseconds per launch and TFLOP/s (GEMM, attention) or
GB/s of algorithmic bytes (LayerNorm, embedding).  With --flush-l2 every launch is timed on its own
after a 256 MiB write that evicts L2; otherwise the N launches run back to back.  Inputs are
seeded normal values made on the device; the numbers measure speed only.  Device memory
stays under about 5 GB, so one case can run under a profiler."""
import argparse
import json
import re

import torch

from decoder_only_transformer_train_b200 import binding as BD
from decoder_only_transformer_train_b200 import synthetic as S


def gemm_cases(ntok, C, V):
    # name, M, N, K, a_mn, b_mn, epilogue (0 bf16 store, 1 f32 store, 2 f32 accumulate,
    # 3 residual add, 4 GELU keeping the pre-activation, 5 GELU grad)
    return [
        ("qkv_fwd", ntok, 3 * C, C, False, False, 0),
        ("proj_fwd", ntok, C, C, False, False, 1),
        ("fc_fwd", ntok, 4 * C, C, False, False, 0),
        ("mproj_fwd", ntok, C, 4 * C, False, False, 1),
        ("mproj_dX", ntok, 4 * C, C, False, True, 0),
        ("fc_dX", ntok, C, 4 * C, False, True, 1),
        ("qkv_dX", ntok, C, 3 * C, False, True, 1),
        ("proj_dX", ntok, C, C, False, True, 0),
        ("mproj_dW", C, 4 * C, ntok, True, True, 2),
        ("fc_dW", 4 * C, C, ntok, True, True, 2),
        ("qkv_dW", 3 * C, C, ntok, True, True, 2),
        ("proj_dW", C, C, ntok, True, True, 2),
        ("proj_fwd_res", ntok, C, C, False, False, 3),
        ("fc_fwd_gelu", ntok, 4 * C, C, False, False, 4),
        ("mproj_fwd_res", ntok, C, 4 * C, False, False, 3),
        ("mproj_dX_gelu", ntok, 4 * C, C, False, True, 5),
        ("head_fwd", ntok, V, C, False, False, 0),
        ("head_dh", ntok, C, V, False, True, 1),
        ("head_dW", V, C, ntok, True, True, 2),
    ]


class Timer:
    def __init__(self, flush: bool):
        self.flush = flush
        self.scrub = torch.empty(64 << 20, dtype=torch.float32, device="cuda") if flush else None

    def __call__(self, fn, iters: int, warmup: int) -> float:
        """Mean milliseconds per launch of fn()."""
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        if not self.flush:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(iters):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / iters
        total = 0.0
        for _ in range(iters):
            self.scrub.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        return total / iters


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--only", default=".*", help="regular expression over case names")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--flush-l2", action="store_true")
    ap.add_argument("--micro-batch", type=int, default=16)
    ap.add_argument("--seq", type=int, default=1024)
    ap.add_argument("--qkv-std", type=float, default=0.5,
                    help="standard deviation of the attention inputs (the model's q and k are near 0.55)")
    ap.add_argument("--json", action="store_true", help="one JSON object per line")
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("opbench needs a CUDA device")
    BD.lib()
    sel = re.compile(args.only)
    B, T, H, hd, C, V = args.micro_batch, args.seq, 12, 64, 768, 50304
    ntok = B * T
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    rnd = lambda *shape, dt=torch.bfloat16: torch.randn(*shape, device=dev, generator=gen).to(dt)
    timer = Timer(args.flush_l2)

    def report(name, ms, **kw):
        rec = {"case": name, "us": round(ms * 1e3, 2), **kw}
        if args.json:
            print(json.dumps(rec), flush=True)
        else:
            extra = " ".join(f"{k}={v}" for k, v in kw.items())
            print(f"{name:12s} {ms * 1e3:9.1f} us  {extra}", flush=True)

    ws = torch.empty(8 * 4 * C * C, dtype=torch.float32, device=dev)
    for name, M, N, K, a_mn, b_mn, epi in gemm_cases(ntok, C, V):
        if not sel.search(name):
            continue
        A = rnd(K, M) if a_mn else rnd(M, K)
        Bm = rnd(K, N) if b_mn else rnd(N, K)
        out = torch.zeros(M, N, dtype=torch.bfloat16 if epi in (0, 4, 5) else torch.float32, device=dev)
        lda, ldb = (M if a_mn else K), (N if b_mn else K)
        if epi <= 2:
            fn = lambda: BD.gemm_bf16(A, Bm, out, M, N, K, lda, ldb, N, a_mn, b_mn, epilogue=epi,
                                      workspace=ws if epi == 2 else None)
        else:
            aux = rnd(M, N, dt=torch.float32 if epi == 3 else torch.bfloat16)
            bias = rnd(N, dt=torch.float32)
            fn = lambda: BD.gemm_bf16_fused(A, Bm, out, M, N, K, lda, ldb, N, a_mn, b_mn, epi, bias=bias,
                                            aux=aux if epi != 4 else None, ld_aux=N,
                                            aux_out=aux if epi == 4 else None, ld_aux_out=N)
        ms = timer(fn, args.iters, args.warmup)
        report(name, ms, M=M, N=N, K=K, tflops=round(2.0 * M * N * K / (ms * 1e-3) / 1e12, 1))
        del A, Bm, out

    if sel.search("attn_fwd") or sel.search("attn_bwd"):
        qkv = (rnd(ntok, 3 * C, dt=torch.float32) * args.qkv_std).to(torch.bfloat16)
        out = torch.empty(ntok, C, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(B * H * T, dtype=torch.float32, device=dev)
        # causal: half of the T x T scores, 4 * hd flops each (QK^T and PV): 2 B T^2 C
        flops_fwd = 2.0 * B * T * T * C
        fwd = lambda: BD.attention_fwd(qkv, out, lse, B, T, H, hd, BD.GPT2_BF16)
        if sel.search("attn_fwd"):
            ms = timer(fwd, args.iters, args.warmup)
            report("attn_fwd", ms, B=B, T=T, H=H, tflops=round(flops_fwd / (ms * 1e-3) / 1e12, 1))
        if sel.search("attn_bwd"):
            fwd()
            dout = rnd(ntok, C)
            Dbuf = torch.empty(B * H * T, dtype=torch.float32, device=dev)
            dqkv = torch.empty_like(qkv)
            bwd = lambda: BD.attention_bwd(qkv, out, dout, lse, Dbuf, dqkv, B, T, H, hd, BD.GPT2_BF16)
            ms = timer(bwd, args.iters, args.warmup)
            # backward: dP, dV, dQ, dK (4 products, twice the forward; the recomputed S not counted)
            report("attn_bwd", ms, B=B, T=T, H=H, tflops=round(2.0 * flops_fwd / (ms * 1e-3) / 1e12, 1))
        del qkv, out, lse

    if sel.search("ln_fwd"):
        x = rnd(ntok, C, dt=torch.float32)
        w, b = rnd(C, dt=torch.float32), rnd(C, dt=torch.float32)
        y = torch.empty(ntok, C, dtype=torch.bfloat16, device=dev)
        mean = torch.empty(ntok, dtype=torch.float32, device=dev)
        rstd = torch.empty_like(mean)
        fn = lambda: BD.layernorm_fwd(x, w, b, y, mean, rstd, ntok, C, BD.GPT2_BF16)
        ms = timer(fn, args.iters, args.warmup)
        nbytes = ntok * C * (4 + 2) + ntok * 8
        report("ln_fwd", ms, N=ntok, C=C, gbs=round(nbytes / (ms * 1e-3) / 1e9, 1))

    if sel.search("embed_fwd") or sel.search("embed_bwd"):
        # Zipf ids over the real vocabulary, as in the training step's synthetic batches
        ids = S.zipf_tokens(7, ntok, 50257)
        tok = torch.from_numpy(ids).cuda()
        distinct = int(len(set(ids.tolist())))
        if sel.search("embed_fwd"):
            wte, wpe = rnd(50257, C, dt=torch.float32), rnd(T, C, dt=torch.float32)
            x = torch.empty(ntok, C, dtype=torch.float32, device=dev)
            fn = lambda: BD.embedding_fwd(tok, wte, wpe, x, B, T, C, 50257)
            ms = timer(fn, args.iters, args.warmup)
            # x written once; each distinct wte row and each wpe row read once
            nbytes = ntok * C * 4 + (distinct + T) * C * 4
            report("embed_fwd", ms, N=ntok, C=C, gbs=round(nbytes / (ms * 1e-3) / 1e9, 1))
            del wte, wpe, x
        if sel.search("embed_bwd"):
            dx0 = rnd(ntok, C, dt=torch.float32)
            dwte = torch.zeros(50257, C, dtype=torch.float32, device=dev)
            dwpe = torch.zeros(T, C, dtype=torch.float32, device=dev)
            ws = torch.empty(BD.embedding_bwd_ws_bytes(ntok, C), dtype=torch.uint8, device=dev)
            fn = lambda: BD.embedding_bwd(tok, dx0, dwte, dwpe, B, T, C, 50257, ws)
            ms = timer(fn, args.iters, args.warmup)
            # dx0 read once; the distinct dwte rows and every dwpe row read and written
            nbytes = ntok * C * 4 + 2 * (distinct + T) * C * 4
            report("embed_bwd", ms, N=ntok, C=C, distinct=distinct, gbs=round(nbytes / (ms * 1e-3) / 1e9, 1))
            del dx0, dwte, dwpe, ws

    for Vc, name in ((V, "classifier"), (50257, "classifier_50257")):
        if not sel.search(name):
            continue
        # lm_head GEMM with the fused softmax partials, loss, dlogits, dh and dW GEMMs; the
        # second case keeps the unpadded vocabulary (an odd column count), for comparison
        ldl = (Vc + 7) // 8 * 8
        h, W = rnd(ntok, C), rnd(Vc, C)
        targets = torch.randint(0, 50257, (ntok,), device=dev, dtype=torch.int32, generator=gen)
        logits = torch.empty(ntok, ldl, dtype=torch.bfloat16, device=dev)
        aux = torch.empty(BD.classifier_aux_floats(ntok, Vc), dtype=torch.float32, device=dev)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        lse = torch.empty(ntok, dtype=torch.float32, device=dev)
        amax = torch.empty(ntok, dtype=torch.int32, device=dev)
        dh = torch.empty(ntok, C, dtype=torch.float32, device=dev)
        dW = torch.zeros(Vc, C, dtype=torch.float32, device=dev)
        fn = lambda: BD.classifier_fwd_bwd(h, W, targets, ntok, Vc, C, logits, ldl, aux, loss, lse, amax, dh, dW)
        ms = timer(fn, args.iters, args.warmup)
        report(name, ms, N=ntok, V=Vc, C=C, tflops=round(6.0 * ntok * Vc * C / (ms * 1e-3) / 1e12, 1))
        del h, W, logits, dW

    if sel.search("sample"):
        # top-k sampling (k = 50, the pages' value) of 64 rows of bf16 logits over the padded vocabulary
        nr, k = 64, 50
        logits = rnd(nr, V)
        rows = torch.arange(nr, dtype=torch.int32, device=dev)
        u = torch.rand(nr, device=dev, generator=gen)
        out = torch.empty(nr, dtype=torch.int32, device=dev)
        fn = lambda: BD.sample_top_k(logits, V, nr, rows, u, nr, 50257, k, BD.GPT2_BF16, out)
        ms = timer(fn, args.iters, args.warmup)
        # each sampled row read once (bf16)
        nbytes = nr * 50257 * 2
        report("sample", ms, rows=nr, k=k, gbs=round(nbytes / (ms * 1e-3) / 1e9, 1))
        del logits

    if sel.search("optimizer"):
        # global norm + clip + AdamW through the model's entry point, on a context with the 124M
        # model's width and vocabulary but two layers (53.5M parameters, about 1.8 GB of state)
        cfg = BD.Config(n_layer=2, n_embd=C, n_head=H, block_size=T, vocab_size=50257, padded_vocab_size=V,
                        max_batch=1, grad_accum_steps=1, precision=BD.GPT2_BF16)
        # the model's work goes to its own (non-default) stream, on which the timer records
        stream = torch.cuda.Stream()
        model = BD.GPT2(cfg, seed=1, stream=stream.cuda_stream)
        g = model.grad_tensor()
        g.normal_(generator=gen)
        torch.cuda.synchronize()
        n = model.num_params
        fn = lambda: model.adamw_step(6e-4, sync_norm=False)
        with torch.cuda.stream(stream):
            ms = timer(fn, args.iters, args.warmup)
        # norm: read g; AdamW: read p, g, m, v, write p, m, v and the bf16 copy of the >= 2-D tensors
        nbytes = 4 * n + 28 * n + 2 * n
        report("optimizer", ms, params=n, gbs=round(nbytes / (ms * 1e-3) / 1e9, 1))
        del g
        model.close()


if __name__ == "__main__":
    main()
