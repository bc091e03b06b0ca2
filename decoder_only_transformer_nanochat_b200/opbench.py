"""Time one kernel of the decoder step in isolation, at the shapes of one
training step of the d20 workload (M = 16 x 2048 tokens, C = 1280, F = 5120,
V = 65536, H = 10), through the op-level C entry points.  Used for per-kernel
timing and for small, single-kernel ncu captures (--tokens shrinks M, and with
it every shape that grows with the tokens, so a capture holds a few GB).

    python -m decoder_only_transformer_nanochat_b200.opbench --op w1_fwd --iters 5
    python -m decoder_only_transformer_nanochat_b200.opbench --op ce --tokens 8192
    python -m decoder_only_transformer_nanochat_b200.opbench --op rmsnorm --tokens 65536
"""
from __future__ import annotations

import argparse
import json

C, F, V, H, T = 1280, 5120, 65536, 10, 2048


def gemm_shapes(M: int) -> dict:
    """name: (M, N, K, a_mn, b_mn, epilogue) of the step's GEMMs for M tokens."""
    return {
        "qkv_fwd": (M, C + 256, C, 0, 0, "STORE"),
        "o_fwd": (M, C, C, 0, 0, "ADD"),
        "w1_fwd": (M, F, C, 0, 0, "RELU2"),
        "w2_fwd": (M, C, F, 0, 0, "ADD"),
        "head_fwd": (M, V, C, 0, 0, "STORE"),
        "w2_dgrad": (M, F, C, 0, 1, "DRELU2"),
        "w1_dgrad": (M, C, F, 0, 1, "STORE"),
        "w1_wgrad": (F, C, M, 1, 1, "STORE_F32"),
        "w2_wgrad": (C, F, M, 1, 1, "STORE_F32"),
        "o_wgrad": (C, C, M, 1, 1, "STORE_F32"),
        "o_dgrad": (M, C, C, 0, 1, "STORE"),
        "qkv_dgrad": (M, C, C + 256, 0, 1, "STORE"),
        "qkv_wgrad": (C + 256, C, M, 1, 1, "STORE_F32"),
        "head_dgrad": (M, C, V, 0, 1, "STORE"),
        "head_wgrad": (V, C, M, 1, 1, "STORE_F32"),
    }


GEMMS = gemm_shapes(16 * 2048)
ROW_OPS = ["rmsnorm", "rmsnorm_bwd", "rope", "rope_bwd"]


def main():
    import torch

    import decoder_only_transformer_nanochat_b200 as nc
    from decoder_only_transformer_nanochat_b200 import build
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True,
                    choices=sorted(GEMMS) + ["attn_fwd", "attn_bwd", "gemm", "ce"] + ROW_OPS)
    ap.add_argument("--tokens", type=int, default=16 * 2048, help="M (a multiple of 2048)")
    ap.add_argument("--heads", type=int, default=H, help="attention: query heads (d20: 10)")
    ap.add_argument("--window", type=int, default=0, help="attention: sliding window (0: causal)")
    ap.add_argument("--shape", default=None, help="for --op gemm: M,N,K,a_mn,b_mn,EPILOGUE")
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--engine", type=int, default=0)
    args = ap.parse_args()
    build.build()
    g = torch.Generator(device="cuda").manual_seed(0)
    st = torch.cuda.current_stream().cuda_stream
    shapes = gemm_shapes(args.tokens)
    B = args.tokens // T

    def prep():  # work before each timed launch, outside the timed region
        pass

    if args.op == "gemm":
        f = args.shape.split(",")
        shapes["gemm"] = (int(f[0]), int(f[1]), int(f[2]), int(f[3]), int(f[4]), f[5])
    if args.op == "ce":
        M = args.tokens
        z = (torch.randn(M * V, device="cuda", generator=g) * 3.0).to(torch.bfloat16)
        z0 = z.clone()
        tgt = torch.randint(0, V, (M,), device="cuda", dtype=torch.int32, generator=g)
        tl = torch.empty(M, device="cuda", dtype=torch.float32)

        def prep():
            z.copy_(z0)  # the op works in place: every launch starts from the same logits

        def run():
            assert nc.nc_softcap_ce(z.data_ptr(), V, tgt.data_ptr(), tl.data_ptr(), M, V, 1.0 / M,
                                    nc.NC_BF16, st) == 0
        flops = 0.0
    elif args.op in shapes:
        m, n, k, a_mn, b_mn, epi = shapes[args.op]
        # drawn in their storage types: the logit-sized operands stay near 4 GB on the device
        A = torch.randn(m * k, device="cuda", generator=g, dtype=torch.bfloat16).mul_(0.05)
        Bm = torch.randn(n * k, device="cuda", generator=g, dtype=torch.bfloat16).mul_(0.05)
        out_f32 = epi in ("STORE_F32", "ACC_F32")
        D = torch.rand(m * n, device="cuda", generator=g, dtype=torch.float32 if out_f32 else torch.bfloat16)
        lda = m if a_mn else k
        ldb = n if b_mn else k
        code = getattr(nc, "NC_EPI_" + epi)

        def run():
            rc = nc.nc_gemm(A.data_ptr(), lda, a_mn, Bm.data_ptr(), ldb, b_mn, D.data_ptr(), n, m, n, k,
                            nc.NC_BF16, code, args.engine, st)
            assert rc == 0, rc
        flops = 2.0 * m * n * k
    elif args.op in ("rmsnorm", "rmsnorm_bwd"):
        M = args.tokens
        x = torch.randn(M * C, device="cuda", generator=g).to(torch.bfloat16)
        y = torch.empty_like(x)
        r = torch.empty(M, device="cuda", dtype=torch.float32)
        assert nc.nc_rmsnorm(x.data_ptr(), y.data_ptr(), r.data_ptr(), M, C, nc.NC_BF16, st) == 0
        if args.op == "rmsnorm":
            def run():
                assert nc.nc_rmsnorm(x.data_ptr(), y.data_ptr(), r.data_ptr(), M, C, nc.NC_BF16, st) == 0
            nbytes = M * (2.0 * C * 2 + 4)
        else:
            dy = torch.randn(M * C, device="cuda", generator=g).to(torch.bfloat16)
            dx = torch.zeros(M * C, device="cuda", dtype=torch.float32)
            dx_t = torch.empty_like(x)

            def run():  # accumulating into the residual-stream gradient, as the step does
                assert nc.nc_rmsnorm_bwd(dy.data_ptr(), y.data_ptr(), r.data_ptr(), dx.data_ptr(),
                                         dx_t.data_ptr(), M, C, 1, nc.NC_BF16, st) == 0
            nbytes = M * (C * (2.0 + 2.0 + 4.0 + 4.0 + 2.0) + 4)
        flops = 0.0
    elif args.op in ("rope", "rope_bwd"):
        from decoder_only_transformer_nanochat_b200 import Model
        model = Model(depth=20, vocab=V, seq=T, dtype="bf16")
        ld = 128 * (H + 2)
        qkv = (torch.randn(B * T * ld, device="cuda", generator=g) * 0.09).to(torch.bfloat16)
        rq = torch.empty(B * T * H, device="cuda", dtype=torch.float32)
        rk = torch.empty(B * T, device="cuda", dtype=torch.float32)
        assert nc.nc_rope_qknorm(model.handle, qkv.data_ptr(), ld, rq.data_ptr(), rk.data_ptr(), B, T, st) == 0
        per_head = 128 * 2.0
        if args.op == "rope":
            qkv0 = qkv.clone()

            def prep():
                qkv.copy_(qkv0)  # in place: every launch starts from the projections

            def run():
                assert nc.nc_rope_qknorm(model.handle, qkv.data_ptr(), ld, rq.data_ptr(), rk.data_ptr(), B, T,
                                         st) == 0
            nbytes = B * T * (H + 1) * (2 * per_head + 4)
        else:
            d0 = (torch.randn(B * T * ld, device="cuda", generator=g) * 0.1).to(torch.bfloat16)
            dqkv = d0.clone()

            def prep():
                dqkv.copy_(d0)

            def run():
                assert nc.nc_rope_qknorm_bwd(model.handle, dqkv.data_ptr(), qkv.data_ptr(), ld, rq.data_ptr(),
                                             rk.data_ptr(), B, T, st) == 0
            nbytes = B * T * (H + 1) * (3 * per_head + 4)
        flops = 0.0
    else:
        Ha = args.heads
        ld = 128 * (Ha + 2)
        qkv = (torch.randn(B * T * ld, device="cuda", generator=g) * 0.09).to(torch.bfloat16)
        O = torch.empty(B * T * Ha * 128, device="cuda", dtype=torch.bfloat16)
        lse = torch.empty(B * Ha * T, device="cuda", dtype=torch.float32)
        rc = nc.nc_attention_fwd(qkv.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, Ha, nc.NC_BF16,
                                 args.engine, st, window=args.window)
        assert rc == 0
        dO = (torch.randn(B * T * Ha * 128, device="cuda", generator=g) * 0.1).to(torch.bfloat16)
        Dr = torch.empty(B * Ha * T, device="cuda", dtype=torch.float32)
        dqkv = torch.empty(B * T * ld, device="cuda", dtype=torch.bfloat16)
        w = args.window if 0 < args.window < T else T
        keys = 0.5 * w * (w + 1.0) + (T - w) * float(w)
        causal = 4.0 * B * Ha * 128 * keys
        if args.op == "attn_fwd":
            def run():
                assert nc.nc_attention_fwd(qkv.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, Ha,
                                           nc.NC_BF16, args.engine, st, window=args.window) == 0
            flops = causal
        else:
            # with the dK/dV scratch, as the model's step runs it
            rc, nbytes = nc.nc_attention_bwd_scratch_bytes(B, T, Ha, args.window)
            assert rc == 0
            scratch = torch.empty(max(nbytes, 16) // 4, device="cuda", dtype=torch.float32)

            def run():
                assert nc.nc_attention_bwd_ex(qkv.data_ptr(), ld, O.data_ptr(), dO.data_ptr(), lse.data_ptr(),
                                              Dr.data_ptr(), scratch.data_ptr(), nbytes, dqkv.data_ptr(), B, T, Ha,
                                              nc.NC_BF16, args.engine, st, window=args.window) == 0
            flops = 2.0 * causal
    prep()
    run()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.iters)]
    for i in range(args.iters):
        prep()
        ev[2 * i].record()
        run()
        ev[2 * i + 1].record()
    torch.cuda.synchronize()
    # a kernel wait that ran out of time makes the timing meaningless: fail loudly
    rc = nc.nc_ops_status(st, 60000)
    if rc != 0:
        raise SystemExit(f"device status after the timed launches: {nc.nc_strerror(rc)}")
    ms = sorted(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.iters))
    med = ms[len(ms) // 2]
    out = {"op": args.op, "tokens": args.tokens, "shape": args.shape, "window": args.window, "median_ms": med,
           "min_ms": ms[0]}
    if flops:
        out["tflops"] = flops / (med / 1000) / 1e12
    if args.op == "ce":
        out["gbs"] = 2.0 * args.tokens * V * 2 / (med / 1000) / 1e9  # z read once, dz written once
    if args.op in ROW_OPS:
        out["gbs"] = nbytes / (med / 1000) / 1e9  # every operand read once, every output written once
    print(json.dumps(out))


if __name__ == "__main__":
    main()
