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
# DRAM traffic of the GEMM engine: ncu dram__bytes_read.sum +
# dram__bytes_write.sum of one launch of each GEMM class on a small case
# (profiles/gemm_traffic_by_class.md), as a ratio to that launch's
# algorithmic operand + result bytes.  The step's traffic per GEMM launch is
# each class's algorithmic bytes times its ratio, averaged over the launches.
# None when no capture covers the kernels as they stand.
GEMM_TRAFFIC_RATIO = {"fwd": 0.88, "dgrad": 0.898, "wgrad": 1.369, "lmhead": 1.368, "ns": 0.942}


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


LM_CHUNK = 32768  # tokens per lm_head + cross-entropy chunk (the library's default)


def gemm_algorithmic_bytes_by_class(depth=DEPTH, batch=B, seq=T, vocab=V, lm_chunk=LM_CHUNK):
    """Operand and result bytes of every GEMM launch of one step, each operand
    read once and each result written once (bf16 2 B, fp32 4 B; a split-K
    weight gradient counts as one fp32 write), summed per launch class:
    fwd, dgrad, wgrad (the block projections), lmhead (three GEMMs per chunk
    of lm_chunk tokens, each reading or accumulating W_lm once per chunk),
    ns (Newton-Schulz).  Returns ({class: bytes}, {class: launches})."""
    d, f, n = 64 * depth, 4 * 64 * depth, batch * seq
    chunks = -(-n // lm_chunk)
    bf, f4 = 2, 4
    fwd = [
        n * d * bf + 3 * d * d * bf + n * 3 * d * bf,          # q|k|v (+ RoPE / QK-norm)
        n * d * bf + d * d * bf + 2 * n * d * f4,              # o-projection + fp32 residual
        n * d * bf + f * d * bf + n * f * bf,                  # MLP up + ReLU^2
        n * f * bf + d * f * bf + 2 * n * d * f4,              # MLP down + fp32 residual
    ]
    dgrad = [
        n * d * bf + d * f * bf + 2 * n * f * bf,              # du = dy W_down, 2 sqrt(a)
        n * f * bf + f * d * bf + n * d * bf,                  # dh = du W_up
        n * d * bf + d * d * bf + n * d * bf,                  # dh = dy W_o
        n * 3 * d * bf + 3 * d * d * bf + n * d * bf,          # dh = dqkv W_qkv
    ]
    wgrad = [
        n * d * bf + n * f * bf + d * f * f4,                  # dW_down
        n * f * bf + n * d * bf + f * d * f4,                  # dW_up
        2 * n * d * bf + d * d * f4,                           # dW_o
        n * 3 * d * bf + n * d * bf + 3 * d * d * f4,          # dW_qkv
    ]
    lm = [n * d * bf + chunks * vocab * d * bf + n * vocab * bf,       # logits
          n * vocab * bf + chunks * vocab * d * bf + n * d * bf,       # dh = dz W
          n * vocab * bf + n * d * bf + chunks * vocab * d * f4]       # dW += dz^T h
    sq, wide = 4 * depth, 2 * depth                           # Newton-Schulz stacks
    ns = 0
    for cnt, m, k in ((sq, d, d), (wide, d, f)):
        x, a = cnt * m * k * bf, cnt * m * m * bf
        ns += 5 * ((x + a) + (a + a) + (a + x + x))         # A = X X^T; B = cA^2 + bA; Y = BX + aX
    nbytes = {"fwd": float(depth * sum(fwd)), "dgrad": float(depth * sum(dgrad)),
              "wgrad": float(depth * sum(wgrad)), "lmhead": float(sum(lm)), "ns": float(ns)}
    launches = {"fwd": 4 * depth, "dgrad": 4 * depth, "wgrad": 4 * depth, "lmhead": 3 * chunks, "ns": 30}
    return nbytes, launches


def gemm_algorithmic_bytes_per_step(depth=DEPTH, batch=B, seq=T, vocab=V):
    """All GEMM classes of gemm_algorithmic_bytes_by_class together.
    Returns (bytes, launches)."""
    nbytes, launches = gemm_algorithmic_bytes_by_class(depth, batch, seq, vocab)
    return float(sum(nbytes.values())), sum(launches.values())


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


def tensor_peak_at(sm_mhz, sms=148):
    """Dense bf16 tcgen05 rate at a given SM clock: 8192 FLOP per clock per
    SM (M128 x N256 x K16 in 128 clocks), in TFLOP/s."""
    return 8192.0 * sms * sm_mhz * 1e6 / 1e12


def gemm_traffic_per_launch(depth=DEPTH, batch=B, seq=T, vocab=V):
    """Modelled DRAM bytes per GEMM launch of one step from the per-class
    ratios of GEMM_TRAFFIC_RATIO (None when no capture covers the kernels)."""
    if not GEMM_TRAFFIC_RATIO:
        return None, "no small-case capture of the current GEMM kernels"
    by_class, _ = gemm_algorithmic_bytes_by_class(depth, batch, seq, vocab)
    total = sum(GEMM_TRAFFIC_RATIO[c] * b for c, b in by_class.items())
    _, launches = gemm_algorithmic_bytes_per_step(depth, batch, seq, vocab)
    return total / launches, ("per-class DRAM/algorithmic ratios from one-launch ncu captures "
                              "(profiles/gemm_traffic_by_class.md) times each class's "
                              "algorithmic bytes in the step")


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
def host_cpu():
    """CPU model name and logical core count of this host."""
    name = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return name, os.cpu_count() or 1


def oracle_attention_seconds(heads, seed=5):
    """Oracle causal attention forward + backward of one row of T = 2048
    tokens with `heads` heads of 128 (the oracle parallelises over heads)."""
    import oracle
    from pretraining_step_b200 import inputs
    d = heads * 128
    qkv = inputs.bf16_normal(seed, (T, 3 * d))
    q = qkv[:, :d].reshape(1, T, heads, 128)
    k = qkv[:, d:2 * d].reshape(1, T, heads, 128)
    v = qkv[:, 2 * d:].reshape(1, T, heads, 128)
    t0 = time.perf_counter()
    o, lse, _ = oracle.attention(q, k, v)
    oracle.attention_bwd(q, k, v, lse, o)
    return time.perf_counter() - t0


def cpu_oracle_sample():
    """Time the oracle on a bounded sample of the workload and convert to the
    workload's tokens/s.  A B = 1, T = 2048 row of depth 20 is far beyond a
    few seconds of fp64 work, so its two parts are timed separately: the
    per-token part (every projection, norm and the loss) from forward +
    backward on a 16-token row, and the part quadratic in T (causal attention
    forward + backward) on one T = 2048 row with as many heads as threads,
    scaled to the step's 32 rows x 20 layers x 10 heads; plus the
    Newton-Schulz of one matrix of each Muon shape, scaled to 80 + 40.  Then
    the same at one thread on a smaller sample."""
    import numpy as np
    import oracle
    from pretraining_step_b200 import inputs
    oracle.lib()
    threads_all = oracle.threads()
    cpu_name, nproc = host_cpu()
    P = inputs.random_params(DEPTH, seed=1)
    t_tok = 16
    tok, tgt = inputs.token_batch(2, 1, t_tok)
    t0 = time.perf_counter()
    oracle.gpt_fwd_bwd(DEPTH, P, tok, tgt)
    fb = time.perf_counter() - t0
    heads = max(1, min(threads_all, 16))
    att = oracle_attention_seconds(heads)
    head_rows = B * DEPTH * (64 * DEPTH // 128)      # (row, layer, head) attention units
    t0 = time.perf_counter()
    oracle.newton_schulz(P[1])                  # one d x d matrix (of 80)
    ns_sq = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.newton_schulz(P[5])                  # one 4d x d matrix (of 40)
    ns_w = time.perf_counter() - t0
    step_s = fb / t_tok * (B * T) + att / heads * head_rows + 4 * DEPTH * ns_sq + 2 * DEPTH * ns_w
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
        att1 = oracle_attention_seconds(1)
        d = 64 * DEPTH
        G = np.asarray(P[1][: d // 2, : d // 2], dtype=np.float64)
        t0 = time.perf_counter()
        oracle.newton_schulz(G)
        ns1 = time.perf_counter() - t0
    finally:
        oracle.threads(threads_all)
    step1_s = fb1 / t1_tok * (B * T) + att1 * head_rows + 4 * DEPTH * 8 * ns1 + \
        2 * DEPTH * 24 * ns1
    return {
        "value": (B * T) / step_s,
        "unit": "tokens/s",
        "cores": threads_all,
        "kind": "oracle",
        "host": {"cpu": cpu_name, "nproc": nproc, "omp_threads": threads_all},
        "sample": ("double-precision CPU oracle on %d threads: per-token part from forward + "
                   "backward of depth 20 on 1 x %d tokens (%.1f s) scaled to 65536 tokens; "
                   "attention forward + backward of one T=2048 row with %d heads (%.1f s) "
                   "scaled to 32 rows x 20 layers x 10 heads; Newton-Schulz of one 1280x1280 "
                   "(%.1f s) and one 5120x1280 matrix (%.1f s) scaled to 80 + 40 matrices"
                   % (threads_all, t_tok, fb, heads, att, ns_sq, ns_w)),
        "sample_seconds": fb + att + ns_sq + ns_w,
        "one_thread": {
            "value": (B * T) / step1_s, "unit": "tokens/s", "cores": 1,
            "sample": ("forward+backward on 1 x %d tokens (%.1f s) scaled to 65536 tokens, "
                       "attention of one T=2048 head (%.1f s) scaled to 6400 head-rows, "
                       "Newton-Schulz of one 640x640 matrix (%.1f s) scaled by FLOPs to "
                       "80 x 1280^2 and 40 x 5120x1280" % (t1_tok, fb1, att1, ns1)),
            "sample_seconds": fb1 + att1 + ns1,
        },
    }


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample of the workload (forward + backward on an 8-token row, the
    attention forward + backward of one T = 2048 row, and the Newton-Schulz
    of one block matrix), converted to the 65536-token step's time."""
    if rank != 0:
        return 0
    from pretraining_step_b200 import inputs
    import oracle
    oracle.lib()
    threads = oracle.threads()
    heads = max(1, min(threads, 16))
    head_rows = B * DEPTH * (64 * DEPTH // 128)
    P = inputs.random_params(DEPTH, seed=1)
    t_tok = 8
    times_fb, times_att, times_ns = [], [], {"sq": [], "w": []}
    for step in range(args.warmup + args.steps):
        tok, tgt = inputs.token_batch(100 + step, 1, t_tok)
        t0 = time.perf_counter()
        oracle.gpt_fwd_bwd(DEPTH, P, tok, tgt)
        fb = time.perf_counter() - t0
        att = oracle_attention_seconds(heads, seed=200 + step)
        which = "sq" if step % 2 == 0 else "w"
        t0 = time.perf_counter()
        oracle.newton_schulz(P[1] if which == "sq" else P[5])
        ns = time.perf_counter() - t0
        if step >= args.warmup:
            times_fb.append(fb)
            times_att.append(att)
            times_ns[which].append(ns)
    fb_tok = float(np.mean(times_fb)) / t_tok
    att_row = float(np.mean(times_att)) / heads
    ns_sq = float(np.mean(times_ns["sq"])) if times_ns["sq"] else 0.0
    ns_w = float(np.mean(times_ns["w"])) if times_ns["w"] else ns_sq * 4.5
    step_s = fb_tok * B * T + att_row * head_rows + 4 * DEPTH * ns_sq + 2 * DEPTH * ns_w
    value = B * T / step_s
    cpu_name, nproc = host_cpu()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(), "global_batch": B, "seq_len": T,
                   "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "host": {"cpu": cpu_name, "nproc": nproc, "omp_threads": threads},
                         "sample": "each step: oracle forward+backward on 1 x %d tokens, "
                                   "attention forward+backward of one T=2048 row with %d "
                                   "heads, and Newton-Schulz of one block matrix (alternating "
                                   "1280x1280 / 5120x1280), scaled to the 65536-token step, "
                                   "6400 attention head-rows and 120 matrices" % (t_tok, heads)},
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

    # The step as one CUDA graph: it reads its token ids from tok_g / tgt_g,
    # refilled on the stream from the resident batches before every replay.
    tok_g = torch.empty_like(toks[0])
    tgt_g = torch.empty_like(tgts[0])
    m.capture_step(tok_g, tgt_g, loss_dev, LR, MOMENTUM)

    def replay(i):
        tok_g.copy_(toks[i % nbat])
        tgt_g.copy_(tgts[i % nbat])
        m.replay_step()

    with torch.cuda.stream(stream):
        replay(0)  # first launch of the instantiated graph, untimed
        m.sync()

    # ---- device-timed region (inputs resident, no per-launch profiling events)
    clocks = ClockSampler(local_rank)
    clocks.start()
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
            replay(i)
            marks[i + 1].record(stream)
        e1.record(stream)
    m.sync()
    torch.cuda.synchronize()
    barrier()
    launches = m.launch_count() - launches0
    ms = e0.elapsed_time(e1)
    clk = clocks.stop()
    ms_max = max_over_ranks(ms, world, dev)
    median_max = max_over_ranks(float(np.median(step_times_ms(marks))), world, dev)
    final_loss = float(loss_dev.item())

    # ---- profiled pass: the same step run eagerly with CUDA events around
    # every launch (on the launch stream), for the per-kernel table only.
    prof_steps = 3
    m.profile(True)
    m.profile_read()  # reset
    pe0 = torch.cuda.Event(enable_timing=True)
    pe1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        pe0.record(stream)
        for i in range(prof_steps):
            step(i)
        pe1.record(stream)
    m.sync()
    torch.cuda.synchronize()
    prof = m.profile_read()
    m.profile(False)
    prof_ms_per_step = pe0.elapsed_time(pe1) / prof_steps

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
    gemm_traffic, traffic_source = gemm_traffic_per_launch()
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
                     "frac_at_step_clock": (gemm_ach / tensor_peak_at(clk["sm_mhz"])
                                            if clk else None),
                     "traffic": gemm_traffic,
                     "traffic_unit": "bytes per launch",
                     "traffic_source": traffic_source,
                     "traffic_algorithmic": gemm_alg_bytes / gemm_alg_launches,
                     "peak_source": peak_kind + " bf16_tflops_sustained",
                     "launches_per_step": g_n / prof_steps, "ms_per_step": g_ms / prof_steps,
                     "share": g_ms / total_ms},
        "kernels_pass": {"steps": prof_steps, "ms_per_step": prof_ms_per_step,
                         "how": "eager steps after the timed region, CUDA events around "
                                "every launch on the launch stream"},
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
    if args.op == "ns_sweep":
        return run_ns_sweep(args, peaks, peak_kind)
    if args.op == "gemm_traffic":
        return run_gemm_traffic(args)
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
        if args.fp8:
            # E4M3 operands (both K-major), quantised once before timing.
            assert ak and bk and K % 16 == 0, "--fp8 needs K-major operands and K a multiple of 16"
            qa = torch.empty(M * K, device="cuda", dtype=torch.uint8)
            qb = torch.empty(N * K, device="cuda", dtype=torch.uint8)
            sc = torch.zeros(2, device="cuda", dtype=torch.float32)
            scratch = torch.zeros(2, device="cuda", dtype=torch.int32)
            quant = lambda: nc.fp8_quantize(A, M, K, qa, sc[0:1], scratch[0:1])
            quant()
            nc.fp8_quantize(Bm, N, K, qb, sc[1:2], scratch[1:2])
            torch.cuda.synchronize()
            ev[0].record()
            for _ in range(3):
                quant()
            ev[1].record()
            torch.cuda.synchronize()
            quant_ms = ev[0].elapsed_time(ev[1]) / 3
            run = lambda: nc.gemm(M, N, K, qa, qb, D, epi=epi, aux=aux,
                                  split_k=0 if epi == nc.EPI_ACC_F32 else 1, ab_scale=sc)
            nbytes -= 1.0 * (M * K + N * K)
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
    line = {"op": args.op, "shape": dims, "ms_per_launch": ms, "tflops": tf,
            "frac_of_burst_peak": tf / peaks["bf16_tflops"],
            "peak_source": peak_kind, "algorithmic_bytes": nbytes}
    if args.op == "gemm" and args.fp8:
        # fp8 peak: the measured bf16 burst peak times the nominal fp8 : bf16 ratio (2).
        line.update({"dtype": "e4m3", "frac_of_burst_peak": tf / (2.0 * peaks["bf16_tflops"]),
                     "peak_note": "measured bf16 burst x 2 (nominal dense fp8 : bf16 ratio)",
                     "quantize_a_ms": quant_ms})
    print(json.dumps(line), flush=True)
    return 0


NS_SWEEP = ((64, 1664, 1664), (26, 1664, 6656), (26, 6656, 1664))


def ns_sweep_flops(stacks=NS_SWEEP, steps=5):
    """Newton-Schulz FLOPs of the sweep: per step and matrix, with m <= n the
    short side, X X^T (2 m^2 n), A A (2 m^3) and B X (2 m^2 n)."""
    tot = 0.0
    for count, rows, cols in stacks:
        m, n = min(rows, cols), max(rows, cols)
        tot += count * steps * (4.0 * m * m * n + 2.0 * m ** 3)
    return tot


def run_ns_sweep(args, peaks, peak_kind):
    """The Muon Newton-Schulz sweep alone: 5 quintic steps on seeded N(0, 1)
    bf16 stacks of 64 x 1664^2, 26 x 1664x6656 and 26 x 6656x1664, each
    Frobenius-normalised first (nc_op_newton_schulz), device-timed."""
    import torch
    from pretraining_step_b200 import binding as nc
    g = torch.Generator(device="cuda")
    stacks = []
    for i, (count, rows, cols) in enumerate(NS_SWEEP):
        g.manual_seed(500 + i)
        x = torch.randn(count, rows, cols, generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty_like(x)
        scratch = torch.empty(nc.newton_schulz_scratch_bytes(count, rows, cols),
                              dtype=torch.uint8, device="cuda")
        stacks.append((count, rows, cols, x, out, scratch))

    def sweep():
        for count, rows, cols, x, out, scratch in stacks:
            nc.newton_schulz(x, out, count, rows, cols, 5, scratch)

    for _ in range(args.warmup):
        sweep()
    nc.op_sync()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.steps):
        sweep()
    ev[1].record()
    nc.op_sync()
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / args.steps
    fl = ns_sweep_flops()
    tf = fl / (ms / 1e3) / 1e12
    print(json.dumps({"op": "ns_sweep", "stacks": [list(t[:3]) for t in stacks],
                      "ms_per_sweep": ms, "tflop_per_sweep": fl / 1e12, "tflops": tf,
                      "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"],
                      "peak_source": peak_kind}), flush=True)
    return 0


def gemm_traffic_cases(ntok, depth=DEPTH, vocab=V):
    """The GEMMs of one layer, the lm_head and one Newton-Schulz stack as the
    step launches them, at ntok tokens: (class, name, M, N, K, a_kmajor,
    b_kmajor, epilogue, algorithmic bytes).  The q|k|v projection runs with
    the plain bf16 store in place of its RoPE + QK-norm epilogue (the same
    operand and result bytes)."""
    from pretraining_step_b200 import binding as nc
    d, f, n = 64 * depth, 4 * 64 * depth, ntok
    bf, f4 = 2, 4
    return [
        ("fwd", "qkv", n, 3 * d, d, 1, 1, nc.EPI_STORE_BF16, n * d * bf + 3 * d * d * bf + n * 3 * d * bf),
        ("fwd", "o_resid", n, d, d, 1, 1, nc.EPI_RESID_F32, n * d * bf + d * d * bf + 2 * n * d * f4),
        ("fwd", "up_relu2", n, f, d, 1, 1, nc.EPI_RELU2, n * d * bf + f * d * bf + n * f * bf),
        ("fwd", "down_resid", n, d, f, 1, 1, nc.EPI_RESID_F32, n * f * bf + d * f * bf + 2 * n * d * f4),
        ("dgrad", "du_relu2bwd", n, f, d, 1, 0, nc.EPI_RELU2_BWD, n * d * bf + d * f * bf + 2 * n * f * bf),
        ("dgrad", "dh_up", n, d, f, 1, 0, nc.EPI_STORE_BF16, n * f * bf + f * d * bf + n * d * bf),
        ("dgrad", "dh_o", n, d, d, 1, 0, nc.EPI_STORE_BF16, n * d * bf + d * d * bf + n * d * bf),
        ("dgrad", "dh_qkv", n, d, 3 * d, 1, 0, nc.EPI_STORE_BF16, n * 3 * d * bf + 3 * d * d * bf + n * d * bf),
        ("wgrad", "dW_down", d, f, n, 0, 0, nc.EPI_ACC_F32, n * d * bf + n * f * bf + d * f * f4),
        ("wgrad", "dW_up", f, d, n, 0, 0, nc.EPI_ACC_F32, n * f * bf + n * d * bf + f * d * f4),
        ("wgrad", "dW_o", d, d, n, 0, 0, nc.EPI_ACC_F32, 2 * n * d * bf + d * d * f4),
        ("wgrad", "dW_qkv", 3 * d, d, n, 0, 0, nc.EPI_ACC_F32, n * 3 * d * bf + n * d * bf + 3 * d * d * f4),
        ("lmhead", "logits", n, vocab, d, 1, 1, nc.EPI_STORE_BF16, n * d * bf + vocab * d * bf + n * vocab * bf),
        ("lmhead", "dh_lm", n, d, vocab, 1, 0, nc.EPI_STORE_BF16, n * vocab * bf + vocab * d * bf + n * d * bf),
        ("lmhead", "dW_lm", vocab, d, n, 0, 0, nc.EPI_ACC_F32, n * vocab * bf + n * d * bf + vocab * d * f4),
    ]


def run_gemm_traffic(args):
    """One launch of each GEMM of the step (gemm_traffic_cases at --shape
    ntok tokens, default 16384) after one untimed launch of each, plus one
    Newton-Schulz call on the square stack, for a one-launch-per-kernel ncu
    capture of DRAM bytes (-k regex:gemm_tc -s <untimed launches>).  Prints
    the launch order with each launch's algorithmic bytes."""
    import torch
    from pretraining_step_b200 import binding as nc
    ntok = int(args.shape.split(",")[0]) if args.shape != "16384,5120,1280" else 16384
    cases = gemm_traffic_cases(ntok)
    bufs = []
    for cls, name, M, N, K, ak, bk, epi, nbytes in cases:
        A = (torch.randn(M * K, device="cuda") * 0.5).to(torch.bfloat16)
        Bm = (torch.randn(N * K, device="cuda") * K ** -0.5).to(torch.bfloat16)
        f32 = epi in (nc.EPI_RESID_F32, nc.EPI_ACC_F32)
        D = torch.zeros(M * N, device="cuda", dtype=torch.float32 if f32 else torch.bfloat16)
        aux = None
        if epi == nc.EPI_RESID_F32:
            aux = torch.randn(M * N, device="cuda")
        elif epi == nc.EPI_RELU2_BWD:
            aux = torch.rand(M * N, device="cuda").to(torch.bfloat16)
        bufs.append((M, N, K, ak, bk, epi, A, Bm, D, aux))
    d = 64 * DEPTH
    cnt = 4 * DEPTH
    X = torch.randn(cnt, d, d, device="cuda").to(torch.bfloat16)
    out = torch.empty_like(X)
    scratch = torch.empty(nc.newton_schulz_scratch_bytes(cnt, d, d), dtype=torch.uint8, device="cuda")

    def run_all():
        for M, N, K, ak, bk, epi, A, Bm, D, aux in bufs:
            nc.gemm(M, N, K, A, Bm, D, a_kmajor=ak, b_kmajor=bk, epi=epi, aux=aux,
                    split_k=0 if epi == nc.EPI_ACC_F32 else 1)
        nc.newton_schulz(X, out, cnt, d, d, 5, scratch)

    run_all()      # untimed: 15 GEMMs + 15 Newton-Schulz GEMMs
    nc.op_sync()
    run_all()      # the captured pass
    nc.op_sync()
    ns_x = cnt * d * d * 2
    ns_a = cnt * d * d * 2
    ns_bytes = [(ns_x + ns_a), (ns_a + ns_a), (ns_a + ns_x + ns_x)] * 5
    order = [(c[0], c[1], c[8]) for c in cases] + \
        [("ns", "ns_%s_%d" % (("XXt", "AA", "BX")[i % 3], i // 3), b) for i, b in enumerate(ns_bytes)]
    print(json.dumps({"op": "gemm_traffic", "tokens": ntok, "untimed_gemm_launches": len(order),
                      "launches": [{"class": c, "name": n, "algorithmic_bytes": b}
                                   for c, n, b in order]}), flush=True)
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
    vocab = args.vocab
    m = nc.GPT(depth, vocab=vocab, seed=1234, all_random=True, stream=stream,
               n_kv_head=args.kv_heads, window=windows, fp8=args.fp8)
    tk, tg = inputs.token_batch(20, Bb, T_, vocab=vocab)
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
    free, total = torch.cuda.mem_get_info()  # the model's buffers are all still held here
    m.close()
    tok_s = Bb * T_ / (ms / 1e3)
    fpt = step_flops_per_token(depth, T_, vocab, args.kv_heads, windows)
    print(json.dumps({"op": "step", "depth": depth, "B": Bb, "T": T_, "vocab": vocab,
                      "kv_heads": args.kv_heads, "device_gb_in_use": (total - free) / 1e9,
                      "gemm_operands": "e4m3 (block projections)" if args.fp8 else "bf16",
                      "device_gb_total": total / 1e9,
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
    ap.add_argument("--op", choices=["gemm", "attn", "attn_bwd", "adamw", "step", "ns_sweep",
                                     "gemm_traffic"],
                    default=None,
                    help="time one kernel class alone instead of the step ('step': the whole "
                         "step of the model --shape depth,B,T with the options below)")
    ap.add_argument("--kv-heads", type=int, default=0, help="--op step: KV heads (0: one per head)")
    ap.add_argument("--window-pattern", default=None,
                    help="--op step: per-layer pattern of S (short window) and L (full causal)")
    ap.add_argument("--short-window", type=int, default=1024, help="--op step: the S window")
    ap.add_argument("--vocab", type=int, default=V,
                    help="--op step: vocabulary (smaller only for kernel captures on a small case)")
    ap.add_argument("--shape", default="16384,5120,1280")
    ap.add_argument("--fp8", action="store_true",
                    help="--op gemm: E4M3 operands (quantised before timing) with per-tensor "
                         "scales; --op step: the model's fp8 mode")
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
