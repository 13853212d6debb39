"""Throughput of the depth-20 nanochat base-pretraining step on B200.

One step = forward + backward of the depth-20 GPT (d 1280, 10 heads x 128,
MLP 5120, vocab 32768) on B = 32 rows of T = 2048 synthetic token ids,
followed by the Muon update of the 120 block matrices.  Weights are
random-init (every matrix drawn, so no branch multiplies zeros); token ids
are uniform SplitMix64 draws (the pages' web-text shards are not available).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line (rank 0).  `value` is device-timed whole-job tokens/s
with inputs resident in HBM; `e2e` is the same metric through the C ABI
with the token ids in pinned host memory, copied in every step, and the
loss read back every step.  N > 1 runs N independent replicas (one process
per GPU under torchrun): the step has no exchange.  --impl reference runs
the CPU oracle on bounded samples of the same workload on the host cores.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "train tokens/s and MFU (bf16 peak) at depth-20 GPT, 1×B200"
DEPTH, B, T, V = 20, 32, 2048, 32768
LR, MOMENTUM = 0.02, 0.95
NOMINAL_BF16_TFLOPS = 2250.0
# DRAM bytes (read + write) per GEMM launch, averaged over the 273 GEMM
# launches of one step of this workload: ncu dram__bytes_read.sum +
# dram__bytes_write.sum, profiles/step_d20_b32_t2048_launches.md.  Valid
# for the GEMM kernels as captured there; set to None when they change.
GEMM_DRAM_BYTES_PER_LAUNCH = 1017.3e6


def model_flops_per_token(depth=DEPTH, seq=T, vocab=V):
    """Algorithmic training FLOPs per token: 6 * N_matmul + 6 * L * d * T
    (causal attention counts the half of QK^T and PV it computes)."""
    d = 64 * depth
    n_mm = 12 * depth * d * d + vocab * d
    return 6.0 * n_mm + 6.0 * depth * d * seq


def step_flops_per_token(depth, seq, vocab, n_kv_head=0, windows=None):
    """model_flops_per_token for the model with grouped KV heads and per-layer
    windows: N_mm = L (10 d^2 + 2 dkv d) + V d, and each layer's attention
    counts the (query, key) band a window of w keys leaves in the causal
    triangle, T w - w^2 / 2 (T^2 / 2 for full causal, the convention of
    6 L d T)."""
    d = 64 * depth
    H = d // 128
    dkv = 128 * (n_kv_head if n_kv_head > 0 else H)
    n_mm = depth * (10 * d * d + 2 * dkv * d) + vocab * d
    attn = 0.0
    for l in range(depth):
        w = seq if windows is None or windows[l] < 0 else min(windows[l], seq)
        attn += 12.0 * d * (seq * w - w * w / 2.0) / seq
    return 6.0 * n_mm + attn


def gemm_algorithmic_bytes_per_step(depth=DEPTH, batch=B, seq=T, vocab=V):
    """Operand and result bytes of every GEMM launch of one step, each operand
    read once and each result written once (bf16 2 B, fp32 4 B; a split-K
    weight gradient counts as one fp32 write).  Returns (bytes, launches)."""
    d, f, n = 64 * depth, 4 * 64 * depth, batch * seq
    bf, f4 = 2, 4
    per_layer = [
        n * d * bf + 3 * d * d * bf + n * 3 * d * bf,          # q|k|v (+ RoPE / QK-norm)
        n * d * bf + d * d * bf + 2 * n * d * f4,              # o-projection + fp32 residual
        n * d * bf + f * d * bf + n * f * bf,                  # MLP up + ReLU^2
        n * f * bf + d * f * bf + 2 * n * d * f4,              # MLP down + fp32 residual
        n * d * bf + d * f * bf + 2 * n * f * bf,              # du = dy W_down, 2 sqrt(a)
        n * f * bf + f * d * bf + n * d * bf,                  # dh = du W_up
        n * d * bf + d * d * bf + n * d * bf,                  # dh = dy W_o
        n * 3 * d * bf + 3 * d * d * bf + n * d * bf,          # dh = dqkv W_qkv
        n * d * bf + n * f * bf + d * f * f4,                  # dW_down
        n * f * bf + n * d * bf + f * d * f4,                  # dW_up
        2 * n * d * bf + d * d * f4,                           # dW_o
        n * 3 * d * bf + n * d * bf + 3 * d * d * f4,          # dW_qkv
    ]
    lm = [n * d * bf + vocab * d * bf + n * vocab * bf,       # logits
          n * vocab * bf + vocab * d * bf + n * d * bf,       # dh = dz W
          n * vocab * bf + n * d * bf + vocab * d * f4]       # dW = dz^T h
    sq, wide = 4 * depth, 2 * depth                           # Newton-Schulz stacks
    ns = 0
    for cnt, m, k in ((sq, d, d), (wide, d, f)):
        x, a = cnt * m * k * bf, cnt * m * m * bf
        ns += 5 * ((x + a) + (a + a) + (a + x + x))         # A = X X^T; B = cA^2 + bA; Y = BX + aX
    total = depth * sum(per_layer) + sum(lm) + ns
    return float(total), depth * len(per_layer) + len(lm) + 30


def max_over_ranks(x, world, device="cpu"):
    """The largest x over the ranks of the default process group (x itself on
    one rank).  Multi-GPU device times are reported as this maximum."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def step_times_ms(marks):
    """Device time of each step from the K + 1 events recorded around and
    between the K timed steps."""
    return [marks[i].elapsed_time(marks[i + 1]) for i in range(len(marks) - 1)]


def replica_tokens_per_s(steps, world, ms_max, batch=B, seq=T):
    """Whole-job throughput of `world` replicas that each ran `steps` steps of
    batch x seq tokens, timed by the slowest rank (ms_max)."""
    return steps * batch * seq * world / (ms_max / 1e3)


def ns_flops(depth=DEPTH):
    """Newton-Schulz FLOPs of one Muon step (5 iterations, m <= n Gram form)."""
    d = 64 * depth
    sq = 2 * d ** 3 * 3                      # X X^T, A A, B X for d x d
    wide = 2 * (d * d * 4 * d) * 2 + 2 * d ** 3  # X X^T and B X at n = 4d, A A at d
    return 5.0 * (4 * depth * sq + 2 * depth * wide)


def workload_name():
    return ("depth-20 GPT (d 1280, 10x128 heads, MLP 5120, vocab 32768), bf16, B=32, T=2048: "
            "forward + backward + Muon step")


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", "nc_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        load = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": float(np.median(load)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle sample
def cpu_oracle_sample(budget_s=20.0, per_step=False):
    """Time the oracle on a bounded sample of the workload and convert to the
    workload's tokens/s: forward+backward on a short row (cost per token) and
    the Newton-Schulz of one matrix of each Muon shape (cost per matrix), on
    all host cores; then the same at one thread on a smaller sample (2
    tokens, one (d/2) x (d/2) Newton-Schulz scaled by its FLOPs)."""
    import numpy as np
    import oracle
    from pretraining_step_b200 import inputs
    oracle.lib()
    threads_all = oracle.threads()
    P = inputs.random_params(DEPTH, seed=1)
    t_tok = 16
    tok, tgt = inputs.token_batch(2, 1, t_tok)
    t0 = time.perf_counter()
    oracle.gpt_fwd_bwd(DEPTH, P, tok, tgt)
    fb = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.newton_schulz(P[1])                  # one d x d matrix (of 80)
    ns_sq = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.newton_schulz(P[5])                  # one 4d x d matrix (of 40)
    ns_w = time.perf_counter() - t0
    step_s = fb / t_tok * (B * T) + 4 * DEPTH * ns_sq + 2 * DEPTH * ns_w
    # One thread.  Newton-Schulz costs 6 n^3 per iteration for an n x n matrix
    # and 18 n^3 for the 4n x n one (4 m n^2 + 2 n^3 with m = 4n), so the
    # (d/2)^2 sample scales by 8 to d x d and by 24 to 4d x d.
    oracle.threads(1)
    try:
        t1_tok = 2
        tok1, tgt1 = inputs.token_batch(3, 1, t1_tok)
        t0 = time.perf_counter()
        oracle.gpt_fwd_bwd(DEPTH, P, tok1, tgt1)
        fb1 = time.perf_counter() - t0
        d = 64 * DEPTH
        G = np.asarray(P[1][: d // 2, : d // 2], dtype=np.float64)
        t0 = time.perf_counter()
        oracle.newton_schulz(G)
        ns1 = time.perf_counter() - t0
    finally:
        oracle.threads(threads_all)
    step1_s = fb1 / t1_tok * (B * T) + 4 * DEPTH * 8 * ns1 + 2 * DEPTH * 24 * ns1
    return {
        "value": (B * T) / step_s,
        "unit": "tokens/s",
        "cores": threads_all,
        "kind": "oracle",
        "sample": ("double-precision CPU oracle on %d threads: forward+backward of depth 20 on "
                   "1 x %d tokens (%.1f s) scaled to 65536 tokens, plus Newton-Schulz of one "
                   "1280x1280 (%.1f s) and one 5120x1280 matrix (%.1f s) scaled to 80 + 40 "
                   "matrices" % (threads_all, t_tok, fb, ns_sq, ns_w)),
        "sample_seconds": fb + ns_sq + ns_w,
        "one_thread": {
            "value": (B * T) / step1_s, "unit": "tokens/s", "cores": 1,
            "sample": ("forward+backward on 1 x %d tokens (%.1f s) scaled to 65536 tokens, "
                       "plus Newton-Schulz of one 640x640 matrix (%.1f s) scaled by FLOPs to "
                       "80 x 1280^2 and 40 x 5120x1280" % (t1_tok, fb1, ns1)),
            "sample_seconds": fb1 + ns1,
        },
    }


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank):
    if rank != 0:
        return 0
    from pretraining_step_b200 import inputs
    import oracle
    oracle.lib()
    P = inputs.random_params(DEPTH, seed=1)
    t_tok = 8
    times_fb, times_ns = [], {"sq": [], "w": []}
    for step in range(args.warmup + args.steps):
        tok, tgt = inputs.token_batch(100 + step, 1, t_tok)
        t0 = time.perf_counter()
        oracle.gpt_fwd_bwd(DEPTH, P, tok, tgt)
        fb = time.perf_counter() - t0
        which = "sq" if step % 2 == 0 else "w"
        t0 = time.perf_counter()
        oracle.newton_schulz(P[1] if which == "sq" else P[5])
        ns = time.perf_counter() - t0
        if step >= args.warmup:
            times_fb.append(fb)
            times_ns[which].append(ns)
    fb_tok = float(np.mean(times_fb)) / t_tok
    ns_sq = float(np.mean(times_ns["sq"])) if times_ns["sq"] else 0.0
    ns_w = float(np.mean(times_ns["w"])) if times_ns["w"] else ns_sq * 4.5
    step_s = fb_tok * B * T + 4 * DEPTH * ns_sq + 2 * DEPTH * ns_w
    value = B * T / step_s
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(), "global_batch": B, "seq_len": T,
                   "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: oracle forward+backward on 1 x %d tokens and "
                                   "Newton-Schulz of one block matrix (alternating 1280x1280 / "
                                   "5120x1280), scaled to the 65536-token step and 120 "
                                   "matrices" % t_tok},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ native arm
def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from pretraining_step_b200 import binding as nc
    from pretraining_step_b200 import inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    peaks, peak_kind = load_peaks()

    m = nc.GPT(DEPTH, vocab=V, seed=1234 + rank, all_random=True, stream=stream)
    # A few distinct batches, resident in HBM.
    nbat = 4
    toks, tgts = [], []
    for i in range(nbat):
        tk, tg = inputs.token_batch(20 + 97 * rank + i, B, T)
        toks.append(torch.from_numpy(tk).to(dev))
        tgts.append(torch.from_numpy(tg).to(dev))
    loss_dev = torch.zeros(1, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()

    def step(i):
        m.fwd_bwd_async(toks[i % nbat], tgts[i % nbat], loss_dev)
        m.muon_step(LR, MOMENTUM)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
        m.sync()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- device-timed region (inputs resident)
    clocks = ClockSampler(local_rank)
    clocks.start()
    m.profile(True)
    m.profile_read()  # reset
    launches0 = m.launch_count()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with torch.cuda.stream(stream):
        e0.record(stream)
        marks[0].record(stream)
        for i in range(args.steps):
            step(i)
            marks[i + 1].record(stream)
        e1.record(stream)
    m.sync()
    torch.cuda.synchronize()
    barrier()
    launches = m.launch_count() - launches0
    ms = e0.elapsed_time(e1)
    prof = m.profile_read()
    m.profile(False)
    clk = clocks.stop()
    ms_max = max_over_ranks(ms, world, dev)
    median_max = max_over_ranks(float(np.median(step_times_ms(marks))), world, dev)
    final_loss = float(loss_dev.item())

    # ---- end-to-end through the C ABI with host buffers
    pin_tok = [torch.from_numpy(inputs.token_batch(20 + 97 * rank + i, B, T)[0]).pin_memory()
               for i in range(nbat)]
    pin_tgt = [torch.from_numpy(inputs.token_batch(20 + 97 * rank + i, B, T)[1]).pin_memory()
               for i in range(nbat)]
    e2e_steps = max(3, args.steps // 2)
    barrier()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for i in range(e2e_steps):
            tk = pin_tok[i % nbat]
            tg = pin_tgt[i % nbat]
            # Host pointers: nc_gpt_fwd_bwd copies them in and returns the loss.
            m.fwd_bwd(tk.numpy(), tg.numpy())
            m.muon_step(LR, MOMENTUM)
        f1.record(stream)
    m.sync()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev)
    m.close()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample()

    if rank != 0:
        return 0
    value = replica_tokens_per_s(args.steps, world, ms_max)
    tflops = value * model_flops_per_token() / 1e12
    # Dominant kernel: the tcgen05 GEMM (largest share of device time).
    total_ms = sum(v["ms"] for v in prof.values()) or 1.0
    kernels = {}
    for name, v in sorted(prof.items(), key=lambda kv: -kv[1]["ms"]):
        ent = {"launches": v["launches"], "ms": round(v["ms"], 3),
               "share": round(v["ms"] / total_ms, 4)}
        if v["flops"] > 0:
            ach = v["flops"] / (v["ms"] / 1e3) / 1e12
            ent.update(achieved_tflops=round(ach, 1),
                       frac=round(ach / peaks["bf16_tflops_sustained"], 3))
        elif v["bytes"] > 0:
            ach = v["bytes"] / (v["ms"] / 1e3) / 1e9
            ent.update(achieved_gbs=round(ach, 1), frac=round(ach / peaks["hbm_gbs"], 3))
        kernels[name] = ent
    # The GEMM engine's launches, over every class it serves (forward, input
    # gradient, weight gradient, lm_head, Newton-Schulz).
    g_fl = sum(v["flops"] for k, v in prof.items() if k.startswith("gemm_"))
    g_ms = sum(v["ms"] for k, v in prof.items() if k.startswith("gemm_")) or 1.0
    g_n = sum(v["launches"] for k, v in prof.items() if k.startswith("gemm_"))
    gemm_ach = g_fl / (g_ms / 1e3) / 1e12
    gemm_alg_bytes, gemm_alg_launches = gemm_algorithmic_bytes_per_step()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "ms_per_step_median": median_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic uniform token ids (SplitMix64), random-init weights",
        "config": {"workload": workload_name(), "global_batch": B * world, "seq_len": T,
                   "parallelism": "replicas" if world > 1 else "single-gpu",
                   "l2": "working set (~55 GB of saved activations per step) far above the "
                         "126 MB L2; no flush needed"},
        "tflops": tflops,
        "mfu": tflops / NOMINAL_BF16_TFLOPS,
        "mfu_vs_measured_sustained": tflops / peaks["bf16_tflops_sustained"],
        "flops_per_token": model_flops_per_token(),
        "muon_ns_tflop_per_step": ns_flops() / 1e12,
        "final_loss": final_loss,
        "roofline": {"kernel": "gemm_tc (all classes)", "bound": "tensor", "achieved": gemm_ach,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": gemm_ach / peaks["bf16_tflops_sustained"],
                     "traffic": GEMM_DRAM_BYTES_PER_LAUNCH,
                     "traffic_unit": "bytes per launch (ncu DRAM read + write, mean over the step's GEMM launches)",
                     "traffic_algorithmic": gemm_alg_bytes / gemm_alg_launches,
                     "peak_source": peak_kind + " bf16_tflops_sustained",
                     "launches": g_n, "ms": g_ms, "share": g_ms / total_ms},
        "kernels": kernels,
        "gpu_launches": int(launches),
        "e2e": {"value": replica_tokens_per_s(e2e_steps, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * B * T * 4, "d2h_bytes_per_step": 8,
                "steps": e2e_steps},
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ single-kernel modes
def run_op(args):
    """Time one kernel class alone (for tuning and ncu captures on a small
    case): --op gemm --shape M,N,K[,a_kmajor,b_kmajor] or --op attn --shape B,T,H."""
    import torch
    from pretraining_step_b200 import binding as nc
    peaks, peak_kind = load_peaks()
    torch.manual_seed(0)
    dims = [int(x) for x in args.shape.split(",")]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if args.op == "step":
        return run_step_variant(args, dims, peaks, peak_kind)
    if args.op == "adamw":
        # AdamW on the depth-20 embedding and lm_head ([V, d] each): HBM-bound.
        m = nc.GPT(DEPTH, vocab=V, seed=7, all_random=True)
        step = lambda: m.adamw_step(0.2, 0.004, 0.8, 0.95, 1e-10, 0.0)
        for _ in range(args.warmup):
            step()
        m.sync()
        ev[0].record()
        for _ in range(args.steps):
            step()
        ev[1].record()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.steps
        n = V * 64 * DEPTH
        nbytes = 2 * n * (16.0 + 12.0) + n * 2.0  # g, m, v, W in; m, v, W out; lm_head bf16
        m.close()
        print(json.dumps({"op": "adamw", "shape": [V, 64 * DEPTH], "ms_per_launch": ms,
                          "gbs": nbytes / (ms / 1e3) / 1e9,
                          "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                          "peak_source": peak_kind, "algorithmic_bytes": nbytes}), flush=True)
        return 0
    if args.op == "gemm":
        M, N, K = dims[:3]
        ak = dims[3] if len(dims) > 3 else 1
        bk = dims[4] if len(dims) > 4 else 1
        epi = dims[5] if len(dims) > 5 else nc.EPI_STORE_BF16
        A = torch.randn(M * K, device="cuda").to(torch.bfloat16)
        Bm = (torch.randn(N * K, device="cuda") * K ** -0.5).to(torch.bfloat16)
        f32_out = epi in (nc.EPI_STORE_F32, nc.EPI_RESID_F32, nc.EPI_ACC_F32)
        D = torch.zeros(M * N, device="cuda", dtype=torch.float32 if f32_out else torch.bfloat16)
        aux = None
        if epi == nc.EPI_RESID_F32:
            aux = torch.randn(M * N, device="cuda")
        elif epi in (nc.EPI_RELU2_BWD, nc.EPI_AXPBY_BF16):
            aux = torch.rand(M * N, device="cuda").to(torch.bfloat16)
        run = lambda: nc.gemm(M, N, K, A, Bm, D, a_kmajor=ak, b_kmajor=bk, epi=epi, aux=aux,
                              split_k=0 if epi == nc.EPI_ACC_F32 else 1)
        flops = 2.0 * M * N * K
        nbytes = 2.0 * (M * K + N * K) + M * N * (4 if f32_out else 2) + \
            (0 if aux is None else aux.numel() * aux.element_size())
    else:
        Bb, T_, H = dims
        d = H * 128
        qkv = torch.randn(Bb * T_ * 3 * d, device="cuda").to(torch.bfloat16).view(Bb * T_, 3 * d)
        o = torch.empty(Bb * T_, d, device="cuda", dtype=torch.bfloat16)
        lse = torch.empty(Bb, H, T_, device="cuda", dtype=torch.float32)
        fwd = lambda: nc.attention_fwd(qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, o, d, lse, Bb,
                                       T_, H)
        if args.op == "attn":
            run = fwd
            flops, nbytes = 4.0 * Bb * H * 128 * T_ * (T_ + 1) / 2, 2.0 * Bb * T_ * 4 * d
        else:
            fwd()
            dout = torch.randn(Bb * T_, d, device="cuda").to(torch.bfloat16)
            dq = torch.empty(Bb * T_, d, device="cuda", dtype=torch.float32)
            dkv = torch.empty(Bb * T_, 2 * d, device="cuda", dtype=torch.bfloat16)
            delta = torch.empty(Bb, H, T_, device="cuda", dtype=torch.float32)
            run = lambda: nc.attention_bwd(qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, o, dout, d,
                                           lse, dq, dkv[:, :d], dkv[:, d:], 2 * d, delta, Bb, T_,
                                           H)
            flops, nbytes = 10.0 * Bb * H * 128 * T_ * (T_ + 1) / 2, 2.0 * Bb * T_ * 7 * d
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    ev[0].record()
    for _ in range(args.steps):
        run()
    ev[1].record()
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / args.steps
    tf = flops / (ms / 1e3) / 1e12
    print(json.dumps({"op": args.op, "shape": dims, "ms_per_launch": ms, "tflops": tf,
                      "frac_of_burst_peak": tf / peaks["bf16_tflops"],
                      "peak_source": peak_kind, "algorithmic_bytes": nbytes}), flush=True)
    return 0


def run_step_variant(args, dims, peaks, peak_kind):
    """The forward + backward + Muon step of any model configuration
    (--shape depth,B,T, grouped KV heads, per-layer windows), inputs
    resident, device-timed on the model's stream."""
    import torch
    from pretraining_step_b200 import binding as nc
    from pretraining_step_b200 import inputs
    depth, Bb, T_ = dims
    windows = None
    if args.window_pattern:
        windows = nc.window_pattern(args.window_pattern, depth, args.short_window)
    stream = torch.cuda.Stream()
    m = nc.GPT(depth, vocab=V, seed=1234, all_random=True, stream=stream,
               n_kv_head=args.kv_heads, window=windows)
    tk, tg = inputs.token_batch(20, Bb, T_)
    tok, tgt = torch.from_numpy(tk).cuda(), torch.from_numpy(tg).cuda()
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()

    def step():
        m.fwd_bwd_async(tok, tgt, loss)
        m.muon_step(LR, MOMENTUM)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
        m.sync()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
    m.sync()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    m.close()
    tok_s = Bb * T_ / (ms / 1e3)
    fpt = step_flops_per_token(depth, T_, V, args.kv_heads, windows)
    print(json.dumps({"op": "step", "depth": depth, "B": Bb, "T": T_, "kv_heads": args.kv_heads,
                      "windows": windows, "ms_per_step": ms, "tokens_per_s": tok_s,
                      "flops_per_token": fpt, "tflops": tok_s * fpt / 1e12,
                      "mfu": tok_s * fpt / 1e12 / NOMINAL_BF16_TFLOPS,
                      "peak_source": peak_kind}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["gemm", "attn", "attn_bwd", "adamw", "step"], default=None,
                    help="time one kernel class alone instead of the step ('step': the whole "
                         "step of the model --shape depth,B,T with the options below)")
    ap.add_argument("--kv-heads", type=int, default=0, help="--op step: KV heads (0: one per head)")
    ap.add_argument("--window-pattern", default=None,
                    help="--op step: per-layer pattern of S (short window) and L (full causal)")
    ap.add_argument("--short-window", type=int, default=1024, help="--op step: the S window")
    ap.add_argument("--shape", default="16384,5120,1280")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.op:
        return run_op(args)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
