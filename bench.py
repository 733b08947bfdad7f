"""Benchmark of the SharQ hot path (sharq_prep + sharq_linear) on B200.

Default workload: the linear stack of one Qwen2.5-7B decoder layer -- qkv
3584 -> 4608 and gate+up 3584 -> 37888 (both with the RMSNorm fused into
sharq_prep), o 3584 -> 3584 and down 18944 -> 3584 (no norm; Student-t input)
-- at T = 1, 64, 1024 and 8192 tokens, i.e. from decode to prefill, the
largest single-GPU configuration.  One step = prep + dual-path GEMM of all 16
layers (4 linears x 4 token counts).  Metric: effective TFLOP/s =
sum(2 T K D) / time, whole job (all ranks); µs per layer, per kernel and per
T are reported beside it.  Other workloads: --workload q_proj (Llama-3.1-8B
q_proj decode, T in {1, 16, 128}) and --workload mlp (Llama-3.1-8B MLP
prefill).

Timing: CUDA events on the launching stream around exactly K steps, barrier
+ synchronize on both sides, max over ranks.  The step's working set (packed
weights alone: 550 MB) is larger than the 126 MB L2, so every step reads its
weights from HBM; smaller workloads rotate through up to 16 weight and
activation copies to the same end.  Each step is replayed from a CUDA graph.

--impl reference times the CPU oracle (the only reference this method has:
the pages ship no code) on a bounded sample of the same workload.
"""
import argparse
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

EPS = 1e-5
WORKLOADS = {"q_proj": "llama3.1-8b q_proj K=4096 D=4096 (prep+linear per T), RMSNorm gamma~U(0.5,1.5)",
             "mlp": "llama3.1-8b MLP prefill: gate/up 4096->14336 (shared prep, RMSNorm), down 14336->4096 "
                    "(Student-t input)",
             "qwen_layer": "qwen2.5-7b decoder-layer linears: qkv 3584->4608 (RMSNorm), o 3584->3584, "
                           "gate+up 3584->37888 (RMSNorm), down 18944->3584 (Student-t input)"}
DEFAULT_T = {"q_proj": [1, 16, 128], "mlp": [2048], "qwen_layer": [1, 64, 1024, 8192]}
METRIC = "prep+dual-GEMM effective TFLOP/s (2TKD)"
NOMINAL_FP4_DENSE_PFLOPS = 9.0   # B200 datasheet, dense; sparse 2x


def gemm_alg_bytes(T, K, D):
    """Algorithmic HBM bytes of one sharq_linear: packed weight (0.59375 B per
    element), prepared activation (0.90625 B per element of the 128-padded
    rows) and the bf16 output."""
    Tp = -(-T // 128) * 128
    return K * D * 0.59375 + Tp * K * 0.90625 + T * D * 2


def prep_alg_bytes(T, K):
    """bf16 read (2 B) + outputs (0.90625 B) per activation element; the
    tile-padding rows T..Tp-1 are neither read nor written."""
    return T * K * (2 + 0.90625)


def gemm_split_k(L):
    """Whether sharq_linear runs this layer as the split-K decode kernel (its
    output tiles cannot fill the GPU) rather than the persistent one; mirrors
    the library's launch rule, for naming the kernel in the report."""
    m = -(-L.T // 128)
    n = L.D // 256 if L.D % 256 == 0 else L.D // 128
    return m * n < 74


def gemm_kernel_name(L):
    """The kernel sharq_linear runs for this layer (SharQ mode, ungrouped),
    by the library's launch rule: split-K decode kernel, CTA-pair prefill
    kernel (two or more 128-row tiles, 256-column tiles), or the one-CTA
    persistent kernel."""
    if gemm_split_k(L):
        return "sharq_gemm_kernel (split-K)"
    if -(-L.T // 128) >= 2 and L.D % 256 == 0:
        return "sharq_gemm_pair_kernel"
    return "sharq_gemm_persistent_kernel"


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch,
# from one ncu capture of this script's default command (the eager step's
# launch), keyed by layer and kernel;
# a prep entry sums its two launches (row statistics + strip quantizer).
# Reset an entry whenever its kernel changes, until it is captured again.
NCU_TRAFFIC = {
    "gate_up_T8192/gemm": 138069504 + 577048832,
    "down_T8192/prep": (310391552 + 3221760) + (311673856 + 109505024),
}


def read_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"sharq_bench_clocks_{os.getpid()}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.err = open(self.path + ".err", "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=self.err)
            time.sleep(0.3)  # let the first sample land before the timed region
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
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(values, device=None):
    """Element-wise max over all ranks of per-rank times (ms): with every rank
    running its own replica (weak scaling), the job takes as long as its
    slowest rank.  Identity with one process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(flops_per_rank, world, ms):
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


def init_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------- CPU oracle ---

ORACLE_T = 64        # token rows of the oracle sample
ORACLE_COLS = 1024   # output columns of each weight in the oracle sample


def oracle_layers(workload):
    """The oracle's bounded sample of a workload: each distinct linear of it
    at T = 64 rows (the decode-batch point of the sweep), whole rows of K,
    against the first 1024 output columns of its weight (packed once, outside
    any timed region: weight packing is not part of a layer's work)."""
    import synthetic
    from oracle import sharq as O
    seen, out = set(), []
    for L in workload_layers(workload, [ORACLE_T]):
        if L.shares:
            continue
        key = (L.K, L.D, L.norm, L.base)
        if key in seen:
            continue
        seen.add(key)
        d = min(ORACLE_COLS, L.D)
        w = synthetic.weights(11 + L.K + L.D, L.K, d)
        out.append({"name": L.name, "K": L.K, "D": d, "q": O.pack_weight(w),
                    "gamma": synthetic.gamma(12, L.K) if L.norm else None,
                    "x": synthetic.activations(13 + L.K, ORACLE_T, L.K, base=L.base)})
    return out


def oracle_step(layers, k):
    """One layer of the sample through the oracle (prep + float64 dual GEMM);
    returns its 2TKD FLOPs."""
    from oracle import sharq as O
    L = layers[k % len(layers)]
    O.linear(O.prep(L["x"], L["gamma"], EPS), L["q"])
    return 2.0 * ORACLE_T * L["K"] * L["D"]


def oracle_sample(workload, seconds=10.0):
    """cpu_baseline: the oracle on the workload's bounded sample, layers in
    turn, until about `seconds` of CPU work."""
    layers = oracle_layers(workload)
    flops, done = 0.0, 0
    t0 = time.perf_counter()
    while True:
        flops += oracle_step(layers, done)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds and done >= len(layers):
            break
    threads = os.environ.get("OMP_NUM_THREADS") or str(len(os.sched_getaffinity(0)))
    names = ", ".join(f"{L['name']} K={L['K']}" for L in layers)
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": int(threads), "kind": "oracle",
            "sample": f"{done} layers ({names}; T={ORACLE_T} rows, first {ORACLE_COLS} output columns of each "
                      f"weight, packed beforehand), {el:.1f} s, numpy float32-emulated prep + float64 BLAS GEMM"}


def run_reference(args, world, rank, budget_s=120.0):
    """Time the oracle as it stands.  One step = one layer of the workload's
    bounded sample (oracle_layers), layers in turn.  Steps stop early once
    `budget_s` seconds of timed CPU work have passed so the run stays within a
    few minutes; the value is the work done over the time taken."""
    if rank != 0:
        return
    layers = oracle_layers(args.workload)
    for k in range(args.warmup):
        oracle_step(layers, k)
    flops, done = 0.0, 0
    t0 = time.perf_counter()
    for k in range(args.steps):
        flops += oracle_step(layers, k)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    v = flops / el / 1e12
    cores = len(os.sched_getaffinity(0))
    sample = f"{done} layers of {', '.join(L['name'] for L in layers)} (T={ORACLE_T}, first {ORACLE_COLS} columns)"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "steps_timed": done, "warmup": args.warmup, "ms_per_step": el / done * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload] + f", T in {tuple(args.T)}", "parallelism": "replicas"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{sample}, {el:.1f} s"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU path -----

class Layer:
    """One linear of a workload: (T, K, D), RMSNorm or not, input model."""

    def __init__(self, name, T, K, D, norm, base="normal", shares_prep_with=None):
        self.name, self.T, self.K, self.D, self.norm, self.base = name, T, K, D, norm, base
        self.shares = shares_prep_with

    @property
    def flops(self):
        return 2.0 * self.T * self.K * self.D


def workload_layers(name, t_list):
    if name == "q_proj":
        return [Layer(f"q_proj_T{t}", t, 4096, 4096, True) for t in t_list]
    if name == "qwen_layer":   # Qwen2.5-7B decoder-layer linears
        out = []
        for t in t_list:
            out += [Layer(f"qkv_T{t}", t, 3584, 4608, True),
                    Layer(f"o_proj_T{t}", t, 3584, 3584, False),
                    Layer(f"gate_up_T{t}", t, 3584, 37888, True),
                    Layer(f"down_T{t}", t, 18944, 3584, False, base="student_t")]
        return out
    if name == "mlp":   # Llama-3.1-8B MLP at prefill: gate/up share one prep, then down
        out = []
        for t in t_list:
            out += [Layer(f"gate_T{t}", t, 4096, 14336, True),
                    Layer(f"up_T{t}", t, 4096, 14336, True, shares_prep_with=f"gate_T{t}"),
                    Layer(f"down_T{t}", t, 14336, 4096, False, base="student_t")]
        return out
    raise ValueError(name)


def kernel_us(fn, n_rot, stream, launches=96):
    """Average duration of one launch of fn(i): a graph of `launches`
    back-to-back launches (rotating inputs), replayed, CUDA events."""
    import torch
    reps = max(1, launches // n_rot)
    fn(0)                       # eager warm-up (library workspaces) before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            for i in range(n_rot):
                fn(i)
    for _ in range(2):
        g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(5):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1e3 / (5 * reps * n_rot)


def graph_kernel_launches(g):
    """Number of kernel nodes in a captured graph (torch.cuda.CUDAGraph made
    with keep_graph=True): the kernels one replay launches.  None if the
    graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        count = 0
        for node in nodes[:n]:
            err, t = rt.cudaGraphNodeGetType(node)
            if err == rt.cudaError_t.cudaSuccess and t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                count += 1
        return count
    except Exception:
        return None


def run_gpu(args, world, rank, local):
    import torch
    import torch.distributed as dist

    import sparse_activation_quantization_b200 as sq
    import synthetic
    from sparse_activation_quantization_b200 import build
    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    layers = workload_layers(args.workload, args.T)
    # inputs resident in HBM; decode shapes rotate through copies so that the
    # working set of consecutive steps exceeds the 126 MB L2
    wbytes = sum(sq.sharq_weight_bytes(L.K, L.D) for L in layers)
    n_rot = max(1, min(16, -(-200_000_000 // max(wbytes, 1))))
    weights = {L.name: [] for L in layers}
    for li, L in enumerate(layers):
        for i in range(n_rot):
            W = torch.from_numpy(synthetic.weights(100 + 31 * li + i, L.K, L.D)).to(torch.bfloat16).to(dev)
            weights[L.name].append(sq.PackedWeight(W, stream=stream))
            del W
    gammas, xs, acts, outs, wss = {}, {}, {}, {}, {}
    for L in layers:
        outs[L.name] = torch.empty((L.T, L.D), dtype=torch.bfloat16, device=dev)
        wss[L.name] = sq.Workspace(L.T, L.K, L.D, device=dev)
        if L.shares:
            continue
        gammas[L.name] = (torch.from_numpy(synthetic.gamma(12, L.K)).to(torch.bfloat16).to(dev)
                          if L.norm else None)
        xs[L.name] = [torch.from_numpy(synthetic.activations(1000 * L.T + i, L.T, L.K, base=L.base))
                      .to(torch.bfloat16).to(dev) for i in range(n_rot)]
        acts[L.name] = sq.PreparedAct(L.T, L.K, device=dev)
    torch.cuda.synchronize()

    def prep(L, i):
        x = xs[L.name]
        acts[L.name].prep(x[i % len(x)], gammas[L.name], EPS, stream=stream)

    def gemm(L, i):
        src = L.shares or L.name
        w = weights[L.name]
        sq.linear(acts[src], w[i % len(w)], out=outs[L.name], ws=wss[L.name], stream=stream)

    FUSED_MAX_T = 32   # include/sharq.h SHARQ_FUSED_MAX_T: one-kernel prep+GEMM

    def fused(L):
        return (args.decode_form == "fused" and not L.shares and L.T <= FUSED_MAX_T
                and not any(M.shares == L.name for M in layers))

    def layer(L, i):
        """one whole layer through the public API: sharq_prep_linear where the
        prepared activation is not shared, else sharq_prep + sharq_linear"""
        if fused(L):
            x, w = xs[L.name], weights[L.name]
            sq.prep_linear(x[i % len(x)], gammas[L.name], EPS, w[i % len(w)], out=outs[L.name],
                           ws=wss[L.name], stream=stream)
        else:
            if not L.shares:
                prep(L, i)
            gemm(L, i)

    def step(i):
        for L in layers:
            layer(L, i)

    for i in range(n_rot):
        step(i)
    torch.cuda.synchronize()
    graphs = []
    for i in range(n_rot):
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=stream):
            step(i)
        g.instantiate()
        graphs.append(g)
    torch.cuda.synchronize()
    # kernels per step, counted in the captured graph (every one of them is
    # this library's: the step issues nothing else)
    launches_per_step = graph_kernel_launches(graphs[0])

    for k in range(args.warmup):
        graphs[k % n_rot].replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = Clocks(local)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for k in range(args.steps):
        graphs[k % n_rot].replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    if world > 1:
        ms = max_over_ranks([ms], dev)[0]
        dist.barrier()
    for L in layers:
        assert wss[L.name].check(stream) == 0, "device-side error"

    # --- per-layer and per-kernel times -------------------------------------
    # Back-to-back calls on one activation copy would find part of it in L2
    # from the previous call (the quantizer walks the rows from the last one
    # back), so the preps and layers alternate between at least two copies.
    n_act = max(n_rot, 2)
    for n in xs:
        while len(xs[n]) < n_act:
            xs[n].append(xs[n][0].clone())
    per = {}
    for L in layers:
        g_us = kernel_us(lambda i, L=L: gemm(L, i), n_rot, stream)
        p_us = None if L.shares else kernel_us(lambda i, L=L: prep(L, i), n_act, stream)
        lay = kernel_us(lambda i, L=L: layer(L, i), n_act, stream)
        per[L.name] = {"T": L.T, "K": L.K, "D": L.D, "fused": fused(L), "layer_us": lay, "gemm_us": g_us,
                       "prep_us": p_us,
                       "layer_tflops": L.flops / (lay * 1e-6) / 1e12,
                       "gemm_tflops": L.flops / (g_us * 1e-6) / 1e12,
                       "gemm_gbs": gemm_alg_bytes(L.T, L.K, L.D) / (g_us * 1e-6) / 1e9,
                       "prep_gbs": None if p_us is None else prep_alg_bytes(L.T, L.K) / (p_us * 1e-6) / 1e9}

    # --- end-to-end through the public API with host buffers ----------------
    hx = {n: torch.from_numpy(synthetic.activations(7, xs[n][0].shape[0], xs[n][0].shape[1])).to(torch.bfloat16)
          .pin_memory() for n in xs}
    hy = {L.name: torch.empty((L.T, L.D), dtype=torch.bfloat16).pin_memory() for L in layers}
    dx = {n: torch.empty_like(xs[n][0]) for n in xs}
    h2d = sum(hx[n].numel() * 2 for n in hx)
    d2h = sum(hy[n].numel() * 2 for n in hy)

    # The copies run on two streams of their own, so that the host link (the
    # bound here: ~1.5 GB per step) carries both directions at once and
    # overlaps the kernels; events keep each buffer's reuse in order (a step's
    # input copy waits for the previous step's prep of that input, a GEMM for
    # the previous step's read-back of its output).
    cs_in, cs_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = {n: torch.cuda.Event() for n in xs}            # input on the device
    ev_used = {n: torch.cuda.Event() for n in xs}          # input read by its prep
    ev_out = {L.name: torch.cuda.Event() for L in layers}  # output written
    ev_read = {L.name: torch.cuda.Event() for L in layers}  # output copied to the host
    seen = set()

    def e2e_step(i):
        for L in layers:
            if not L.shares:
                with torch.cuda.stream(cs_in):
                    if L.name in seen:
                        cs_in.wait_event(ev_used[L.name])
                    dx[L.name].copy_(hx[L.name], non_blocking=True)
                    ev_in[L.name].record(cs_in)
                stream.wait_event(ev_in[L.name])
            if L.name in seen:
                stream.wait_event(ev_read[L.name])
            if fused(L):
                w = weights[L.name]
                sq.prep_linear(dx[L.name], gammas[L.name], EPS, w[i % len(w)], out=outs[L.name],
                               ws=wss[L.name], stream=stream)
                ev_used[L.name].record(stream)
            else:
                if not L.shares:
                    acts[L.name].prep(dx[L.name], gammas[L.name], EPS, stream=stream)
                    ev_used[L.name].record(stream)
                gemm(L, i)
            ev_out[L.name].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(ev_out[L.name])
                hy[L.name].copy_(outs[L.name], non_blocking=True)
                ev_read[L.name].record(cs_out)
            seen.add(L.name)
    for i in range(3):
        e2e_step(i % n_rot)
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 50))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    cs_in.wait_stream(stream)
    cs_out.wait_stream(stream)
    for k in range(e2e_steps):
        e2e_step(k % n_rot)
    stream.wait_stream(cs_in)
    stream.wait_stream(cs_out)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    if world > 1:
        e2e_ms = max_over_ranks([e2e_ms], dev)[0]

    # --- every activation mode of the library on one layer: prep + GEMM time,
    # and the relative Frobenius error of Y (float32 output) against the
    # unquantized float32 product Xn W (weight quantization included, the
    # same for every mode) on the first input copy
    MODES = {"sharq": sq.SHARQ_MODE_SHARQ, "nvfp4": sq.SHARQ_MODE_NVFP4, "sharq_per_token": sq.SHARQ_MODE_SHARQ_TOKEN,
             "sparse_only": sq.SHARQ_MODE_SPARSE_ONLY, "dense_dense": sq.SHARQ_MODE_DENSE_DENSE,
             "sparse_sparse": sq.SHARQ_MODE_SPARSE_SPARSE, "sharq_mxfp4": sq.SHARQ_MODE_MXFP4,
             "mxfp4": sq.SHARQ_MODE_MXFP4_PLAIN}
    MX_MODES = (sq.SHARQ_MODE_MXFP4, sq.SHARQ_MODE_MXFP4_PLAIN)

    def mode_table(L, li, src, W0):
        x0 = xs[src][0].float()
        if gammas[src] is not None:
            ss = (xs[src][0].double() ** 2).sum(dim=1)
            inv = (1.0 / torch.sqrt(ss / L.K + float(torch.tensor(EPS, dtype=torch.float32)))).float()
            xn = ((x0 * inv[:, None]) * gammas[src].float()).to(torch.bfloat16).float()
        else:
            xn = x0
        torch.backends.cuda.matmul.allow_tf32 = False  # a true float32 reference product
        yref = xn @ W0.float()
        y32 = torch.empty((L.T, L.D), dtype=torch.float32, device=dev)
        out = {}
        w_mx = None
        for name, mode in MODES.items():
            try:
                a_m = sq.PreparedAct(L.T, L.K, mode=mode, device=dev)
            except Exception as e:  # a shape the mode does not support
                out[name] = {"unsupported": str(e)}
                continue
            if mode in MX_MODES:  # the MXFP4 payloads of the same weights (same rotation)
                if w_mx is None:
                    w_mx = []
                    for i in range(n_rot):
                        Wi = torch.from_numpy(synthetic.weights(100 + 31 * li + i, L.K, L.D)).to(torch.bfloat16).to(dev)
                        w_mx.append(sq.PackedWeight(Wi, stream=stream, fmt=sq.SHARQ_FMT_MXFP4))
                        del Wi
                wsel = lambda i: w_mx[i]
            else:
                wsel = lambda i: weights[L.name][i]
            us = kernel_us(lambda i: (a_m.prep(xs[src][i], gammas[src], EPS, stream=stream),
                                      sq.linear(a_m, wsel(i), out=outs[L.name], ws=wss[L.name],
                                                stream=stream)), n_rot, stream)
            a_m.prep(xs[src][0], gammas[src], EPS, stream=stream)
            sq.linear(a_m, wsel(0), out_dtype=torch.float32, out=y32, ws=wss[L.name], stream=stream)
            torch.cuda.synchronize()
            err = (torch.linalg.norm(y32 - yref) / torch.linalg.norm(yref)).item()
            out[name] = {"layer_us": round(us, 3), "y_rel_err": round(err, 5)}
            del a_m
        return out

    # --- comparators on the same box: plain NVFP4 (dense FP4 GEMM only, same    # --- comparators on the same box: plain NVFP4 (dense FP4 GEMM only, same
    # kernels in SHARQ_MODE_NVFP4) and bf16 cuBLAS (torch.matmul) ---------
    comparators = None
    if args.compare:
        comparators = {}
        for li, L in enumerate(layers):
            act_n = sq.PreparedAct(L.T, L.K, mode=sq.SHARQ_MODE_NVFP4, device=dev)
            src = L.shares or L.name
            xn_ = xs[src][0]
            nv = kernel_us(lambda i, L=L: (act_n.prep(xs[src][i], gammas[src], EPS, stream=stream),
                                           sq.linear(act_n, weights[L.name][i], out=outs[L.name], ws=wss[L.name],
                                                     stream=stream)), n_rot, stream)
            Wb = [torch.from_numpy(synthetic.weights(100 + 31 * li + i, L.K, L.D)).to(torch.bfloat16).to(dev)
                  for i in range(min(n_rot, 2))]
            ob = torch.empty((L.T, L.D), dtype=torch.bfloat16, device=dev)
            bf = kernel_us(lambda i, L=L: torch.matmul(xs[src][i], Wb[i % len(Wb)], out=ob), n_rot, stream)
            comparators[L.name] = {"sharq_layer_us": round(per[L.name]["layer_us"], 3),
                                   "nvfp4_layer_us": round(nv, 3), "bf16_cublas_us": round(bf, 3),
                                   "modes": mode_table(L, li, src, Wb[0])}
            del Wb, act_n

    flops_step = sum(L.flops for L in layers)
    peak_gbs, peak_kind = read_peaks()
    from sparse_activation_quantization_b200 import peak
    pk = peak.fp4_peaks()
    eff_tflops = pk["effective_pflops"] * 1e3
    nominal_eff = 1e3 / (1.0 / NOMINAL_FP4_DENSE_PFLOPS + 1.0 / (2 * NOMINAL_FP4_DENSE_PFLOPS))
    # dominant kernel: the GEMM with the largest share of the step, against
    # the roofline that bounds it (the slower of its tensor time at the
    # combined FP4 peak and its HBM time at the copy bandwidth)
    dom = max(layers, key=lambda L: per[L.name]["gemm_us"])
    t_tensor = dom.flops / (eff_tflops * 1e12)
    t_hbm = gemm_alg_bytes(dom.T, dom.K, dom.D) / (peak_gbs * 1e9)
    gemm_kernel = gemm_kernel_name(dom)
    if t_tensor >= t_hbm:
        ach = per[dom.name]["gemm_tflops"]
        roof = {"kernel": f"{gemm_kernel} ({dom.name})", "bound": "tensor", "achieved": ach, "peak": eff_tflops,
                "unit": "TFLOP/s", "frac": ach / eff_tflops,
                "peak_kind": "measured tcgen05 FP4 dual-GEMM effective (dense %.2f, sparse %.2f PFLOP/s, best of "
                             "1-CTA and 2-CTA forms)" % (pk["dense_pflops"], pk["sparse_pflops"]),
                "frac_of_nominal": ach / nominal_eff,
                "traffic": NCU_TRAFFIC.get(f"{dom.name}/gemm")}
    else:
        ach = per[dom.name]["gemm_gbs"]
        roof = {"kernel": f"{gemm_kernel} ({dom.name})", "bound": "hbm", "achieved": ach, "peak": peak_gbs,
                "unit": "GB/s", "frac": ach / peak_gbs, "peak_kind": peak_kind + " burst copy",
                "traffic": NCU_TRAFFIC.get(f"{dom.name}/gemm")}
    # the prep with the largest share, against HBM
    pdom = max((L for L in layers if per[L.name]["prep_us"] is not None), key=lambda L: per[L.name]["prep_us"])
    pach = per[pdom.name]["prep_gbs"]
    roof_prep = {"kernel": f"sharq_prep ({pdom.name})", "bound": "hbm", "achieved": pach, "peak": peak_gbs,
                 "unit": "GB/s", "frac": pach / peak_gbs, "peak_kind": peak_kind + " burst copy",
                 "traffic": NCU_TRAFFIC.get(f"{pdom.name}/prep")}
    line = None
    if rank == 0:
        ms_step = ms / args.steps
        value = job_tflops(flops_step, world, ms_step)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3 block scales, fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload] + f", T in {tuple(args.T)}",
                       "l2": (f"inputs larger than L2: {n_rot} rotating weight/activation copies"
                              if n_rot > 1 else "working set larger than L2"),
                       "parallelism": "replicas" if world > 1 else "single",
                       "decode_form": ("sharq_prep_linear (one kernel for T <= 32)" if args.decode_form == "fused"
                                       else "sharq_prep + sharq_linear")},
            "layers": {n: {k: (round(v, 3) if isinstance(v, float) else v) for k, v in d.items()}
                       for n, d in per.items()},
            "roofline": roof,
            "roofline_prep": roof_prep,
            "comparators": comparators,
            "e2e": {"value": job_tflops(flops_step, world, e2e_ms), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
            "gpu_launches_per_step": launches_per_step,
            "clocks": clk,
        }
    if world > 1:
        graphs.clear()
        dist.barrier()
        dist.destroy_process_group()
    return line


def run_epilogues(args):
    """Fused preceding-op epilogues against the unfused framework ops, per call
    (CUDA events over graph-replayed back-to-back calls): the SwiGLU product of
    a down projection's input (K = 14336, no RMSNorm, h written out) and the
    residual-stream add before an RMSNorm prep (K = 4096, h written out)."""
    import torch
    import sparse_activation_quantization_b200 as sq
    import synthetic
    from sparse_activation_quantization_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    out = {}
    for T in args.T:
        K = 14336
        g = torch.from_numpy(synthetic.activations(1, T, K) * np.float32(0.5)).to(torch.bfloat16).to(dev)
        u = torch.from_numpy(synthetic.activations(2, T, K, base="student_t")).to(torch.bfloat16).to(dev)
        h = torch.empty_like(u)
        act = sq.PreparedAct(T, K, device=dev)
        fused = kernel_us(lambda i: act.prep_silu_mul(g, u, h, None, EPS, stream=stream), 1, stream, launches=32)
        unfused = kernel_us(lambda i: act.prep(torch.mul(torch.nn.functional.silu(g), u, out=h), None, EPS,
                                               stream=stream), 1, stream, launches=32)
        prep_h = kernel_us(lambda i: act.prep(h, None, EPS, stream=stream), 1, stream, launches=32)
        K2 = 4096
        x = torch.from_numpy(synthetic.activations(3, T, K2)).to(torch.bfloat16).to(dev)
        res = torch.from_numpy(synthetic.activations(4, T, K2)).to(torch.bfloat16).to(dev)
        gam = torch.from_numpy(synthetic.gamma(5, K2)).to(torch.bfloat16).to(dev)
        hr = torch.empty_like(res)
        act2 = sq.PreparedAct(T, K2, device=dev)
        rfused = kernel_us(lambda i: act2.prep_residual(x, res, hr, gam, EPS, stream=stream), 1, stream, launches=32)
        runfused = kernel_us(lambda i: act2.prep(torch.add(x, res, out=hr), gam, EPS, stream=stream), 1, stream,
                             launches=32)
        out[f"T{T}"] = {"silu_mul_fused_us": round(fused, 2), "silu_mul_torch_plus_prep_us": round(unfused, 2),
                        "prep_of_h_us": round(prep_h, 2), "residual_fused_us": round(rfused, 2),
                        "residual_torch_plus_prep_us": round(runfused, 2)}
    print(json.dumps({"epilogues": out, "K_silu": 14336, "K_residual": 4096}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="sharq", choices=["sharq", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--workload", default="qwen_layer", choices=["q_proj", "mlp", "qwen_layer"])
    ap.add_argument("--compare", action="store_true",
                    help="also time plain NVFP4 and bf16 cuBLAS on the same layers")
    ap.add_argument("--T", type=int, nargs="+", default=None)
    ap.add_argument("--epilogues", action="store_true",
                    help="time the fused SwiGLU / residual-add preps against the unfused framework ops")
    ap.add_argument("--decode-form", default="two", choices=["two", "fused"],
                    help="T <= 32 layers: sharq_prep + sharq_linear (two) or sharq_prep_linear's single kernel")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.T is None:
        args.T = DEFAULT_T[args.workload]
    world, rank, local = init_dist(args)
    if args.epilogues:
        if args.T == DEFAULT_T[args.workload]:
            args.T = [1, 16, 128, 2048, 8192]
        run_epilogues(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = oracle_sample(args.workload, args.cpu_seconds)   # before any CUDA work
    line = run_gpu(args, world, rank, local)
    if rank == 0 and line is not None:
        line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
