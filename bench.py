"""Benchmark of the DF-SSM scaffold + LoRA linear stack on B200.

One step = one pass of the whole path over the 48-layer Mamba-2-1.3B
in_proj/out_proj stack (96 linears, one dfssm_linear_stack_fwd call):
activation quantisation + LoRA down-projection, scaffold contraction, LoRA
up-projection and dequantisation, for every linear.

Default workload: the stack at M = 1 token (metric: effective HBM GB/s and
tokens/s). The same line carries the M = 2048 prefill pass (int8 tensor-core
TOPS) under "prefill". Inputs are seeded synthetic tensors with the shapes and
distributions of the Mamba-2-1.3B stack; two independent weight sets are
alternated so that consecutive steps never find their weights in L2.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU (launched by torchrun): every rank runs an independent replica on its
own data (the layer has no exchange step); value = all ranks' work / max time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dfssm_synth as synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0          # nominal dense int8 : bf16 tensor throughput (4.5 : 2.25 PFLOP/s)


# --------------------------------------------------------------------------- work accounting

def stack_bytes(shapes, m):
    """Algorithmic bytes of one stack pass: 1-bit signs, int8 LoRA, fp32 scales, bf16 x in, bf16 y out."""
    sign = sum(d_out * d_in // 8 for d_in, d_out in shapes)
    lora = sum(16 * (d_out + d_in) for d_in, d_out in shapes)
    scales = sum(4 * (2 * d_out + 16) for d_in, d_out in shapes)
    act = sum(2 * m * (d_in + d_out) for d_in, d_out in shapes)
    return sign + lora + scales + act


def stack_ops(shapes, m):
    """Integer ops of one pass: 2*M*d_in*d_out scaffold + 2*M*16*(d_in + d_out) LoRA."""
    return sum(2 * m * d_in * d_out + 2 * m * 16 * (d_in + d_out) for d_in, d_out in shapes)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), src="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=1400.0, src="fallback")


# The source files each measured kernel is built from (its .cu, the shared device headers and the
# host code that fixes its launch); a traffic record stays valid while these files are unchanged.
KERNEL_SOURCES = {
    "decode_kernel": ["decode.cu", "quant.cu", "epilogue.cuh", "ptx.cuh", "dfssm_internal.cuh", "dfssm_api.cu"],
    "prefill_kernel": ["prefill.cu", "quant_rows.cu", "epilogue.cuh", "ptx.cuh", "dfssm_internal.cuh",
                       "dfssm_api.cu"],
    "lm_head_kernel": ["int8_table.cu", "epilogue.cuh", "ptx.cuh", "dfssm_internal.cuh", "dfssm_api.cu"],
    "ssm_step_kernel": ["ssm_step.cu", "epilogue.cuh", "dfssm_internal.cuh"],
}


def kernel_source_hash(names=None):
    """sha256 (16 hex digits) over the named files of the library's csrc/ (all of them by default)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_gemv_gemm_dfssm_b200", "csrc")
    for name in sorted(names if names is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per call from the committed ncu summary, if its kernel's sources are unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    rec = j.get(workload)
    if not rec or rec.get("kernel") not in KERNEL_SOURCES:
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash(KERNEL_SOURCES[rec["kernel"]]):
        return None
    return rec.get("dram_bytes_per_call")


# --------------------------------------------------------------------------- distributed helpers

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, dist, device=None) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist, device=None) -> float:
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Each replica draws its own inputs: the master seed offset by the rank."""
    return synth.MASTER_SEED + 1000003 * rank


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._th = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._th is not None:
            self._th.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- CPU oracle (baseline arms)

def oracle_stack_pass(shapes, m, seed, cfg, linear_ids, threads=0):
    """Run the oracle over the given linears of the stack; returns (seconds, bytes, threads)."""
    import oracle
    inputs = []
    for i in linear_ids:
        d_in, d_out = shapes[i]
        inputs.append((synth.linear_weights(seed, synth.weight_cfg(cfg), i, d_in, d_out),
                       synth.activations(seed, cfg, i, m, d_in), d_in, d_out))
    t0 = time.perf_counter()
    for w, x, d_in, d_out in inputs:
        oracle.linear(x, w, m, d_in, d_out, threads=threads)
    dt = time.perf_counter() - t0
    nbytes = stack_bytes([shapes[i] for i in linear_ids], m)
    return dt, nbytes


def cpu_baseline_leg(shapes, m, seed, cfg, n_single=8):
    """The oracle as it stands on the host cores: the +-1 unpack timed apart, then the forward
    pass from the unpacked weights on every linear with all cores and on the first n_single
    linears single-threaded."""
    import oracle
    inputs = []
    for i, (d_in, d_out) in enumerate(shapes):
        inputs.append((synth.linear_weights(seed, synth.weight_cfg(cfg), i, d_in, d_out),
                       synth.activations(seed, cfg, i, m, d_in), d_in, d_out))
    t0 = time.perf_counter()
    unpacked = [oracle.unpack_sign(w["sign"], d_out, d_in) for w, _, d_in, d_out in inputs]
    t_unpack = time.perf_counter() - t0
    t0 = time.perf_counter()
    for (w, x, d_in, d_out), wpm in zip(inputs, unpacked):
        oracle.linear_unpacked(x, wpm, w, m, d_in, d_out, threads=0)
    t_all = time.perf_counter() - t0
    ns = min(n_single, len(shapes))
    t0 = time.perf_counter()
    for (w, x, d_in, d_out), wpm in list(zip(inputs, unpacked))[:ns]:
        oracle.linear_unpacked(x, wpm, w, m, d_in, d_out, threads=1)
    t_one = time.perf_counter() - t0
    b_all = stack_bytes(shapes, m)
    b_one = stack_bytes(shapes[:ns], m)
    return {"kind": "oracle", "value": b_all / t_all / 1e9, "unit": "GB/s", "cores": oracle_threads(),
            "sample": f"all {len(shapes)} linears at M={m}, forward from unpacked +-1 weights (OpenMP over "
                      f"tokens x rows); the unpack of all linears took {t_unpack:.2f} s and is not in the value",
            "single_thread": {"value": b_one / t_one / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"the first {ns} linears at M={m}, one thread"},
            "unpack_s": t_unpack}


def oracle_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, wl_name):
    """The oracle as it stands, timed on the host cores: each step one forward pass over the
    workload's linears from the unpacked +-1 weights (the unpack is done once, untimed, as in
    the GPU arm's cpu_baseline); for more than 64 tokens a bounded token sample."""
    import oracle
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    wl = synth.WORKLOADS[wl_name]
    shapes, m, cfg = wl["shapes"], wl["m"], wl["cfg"]
    m_s = m if m <= 64 else 4
    cores = oracle_threads()
    inputs = []
    for i, (d_in, d_out) in enumerate(shapes):
        w = synth.linear_weights(synth.MASTER_SEED, synth.weight_cfg(cfg), i, d_in, d_out)
        inputs.append((w, oracle.unpack_sign(w["sign"], d_out, d_in), synth.activations(synth.MASTER_SEED, cfg, i, m_s, d_in),
                       d_in, d_out))

    def one_pass():
        t0 = time.perf_counter()
        for w, wpm, x, d_in, d_out in inputs:
            oracle.linear_unpacked(x, wpm, w, m_s, d_in, d_out, threads=0)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        one_pass()
    tot_t = sum(one_pass() for _ in range(args.steps))
    nb = stack_bytes(shapes, m_s) * args.steps
    gbs = nb / tot_t / 1e9
    sample = (f"all {len(shapes)} linears at M={m_s} per step" + ("" if m_s == m else f" (of M={m})") +
              ", forward from unpacked +-1 weights, OpenMP over tokens x rows")
    line = {
        "impl": "reference", "metric": metric_name(), "value": gbs, "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/int32/f64",
        "data": "synthetic (seeded)", "config": {"workload": wl_name, "m": m, "linears": len(shapes)},
        "cpu_baseline": {"kind": "oracle", "value": gbs, "unit": "GB/s", "cores": cores, "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def metric_name():
    return "effective HBM GB/s and tokens/s for 48-layer in/out_proj stack at M=1; TOPS at M=2048"


# --------------------------------------------------------------------------- GPU arm

def device_weight_sets(shapes, cfg, seed, n_sets=2):
    """n_sets independent weight sets of the stack on the device (alternated so steps miss L2)."""
    import torch
    sets = []
    for s in range(n_sets):
        ws = []
        for i, (d_in, d_out) in enumerate(shapes):
            w = synth.linear_weights(seed + 7919 * s, synth.weight_cfg(cfg), i, d_in, d_out)
            ws.append({k: torch.from_numpy(v).cuda() for k, v in w.items()})
        sets.append(ws)
    return sets


def mapped_address(host_ptr):
    """The device address of pinned host memory (under unified addressing the same number);
    raises, before anything is launched, if the memory is not mapped for the device."""
    from cuda.bindings import runtime as rt
    err, attr = rt.cudaPointerGetAttributes(host_ptr)
    if err != rt.cudaError_t.cudaSuccess or attr.type != rt.cudaMemoryType.cudaMemoryTypeHost or not attr.devicePointer:
        raise RuntimeError(f"host buffer {host_ptr:#x} is not pinned and mapped for the device ({err})")
    return int(attr.devicePointer)


class StackRunner:
    """Device buffers, plan and stack entries for one workload, two weight sets."""

    def __init__(self, shapes, m, cfg, seed, n_sets=2, weight_sets=None):
        import torch
        import bit_gemv_gemm_dfssm_b200 as dfssm
        self.torch, self.dfssm = torch, dfssm
        self.shapes, self.m, self.cfg = shapes, m, cfg
        n = len(shapes)
        self.plan = dfssm.dfssm_linear_plan([(d_in, d_out, m, dfssm.DFSSM_BF16) for d_in, d_out in shapes])
        # contiguous activation buffers (one H2D and one D2H copy per step end to end)
        self.x_off, self.y_off = [], []
        xo = yo = 0
        for d_in, d_out in shapes:
            self.x_off.append(xo)
            self.y_off.append(yo)
            xo += m * d_in
            yo += m * d_out
        self.x_elems, self.y_elems = xo, yo
        self.x_host = torch.empty(xo, dtype=torch.int16).pin_memory()
        xh = self.x_host.numpy().view(np.uint16)
        for i, (d_in, d_out) in enumerate(shapes):
            synth.activations(seed, cfg, i, m, d_in, out=xh[self.x_off[i]:self.x_off[i] + m * d_in].reshape(m, d_in))
        self.x = self.x_host.cuda()
        self.y = torch.empty(yo, dtype=torch.bfloat16, device="cuda")
        self.y_host = torch.empty(yo, dtype=torch.int16).pin_memory()
        if weight_sets is None:
            weight_sets = device_weight_sets(shapes, cfg, seed, n_sets)
        self.sets = [(ws, self.entries(ws, self.y.data_ptr())) for ws in weight_sets[:n_sets]]
        self.n = n
        torch.cuda.synchronize()

    def entries(self, ws, y_base):
        """The device array of stack entries for the weight set ws, entry i's y at y_base plus its
        offset in the contiguous output (y_base: any address the GPU can write)."""
        dfssm = self.dfssm
        ents = [dfssm.StackEntry(dfssm.weights_struct(w["sign"], w["alpha"], w["wa"], w["sa"], w["wb"], w["sb"]),
                                 self.x.data_ptr() + 2 * self.x_off[i], y_base + 2 * self.y_off[i],
                                 dfssm.Debug(0, 0, 0, 0), i, 0) for i, w in enumerate(ws)]
        return self.torch.frombuffer(bytearray(dfssm.stack_entries_bytes(ents)), dtype=self.torch.uint8).cuda()

    def weights_of(self, s):
        return self.sets[s][0]

    def call(self, s, stream):
        self.dfssm.dfssm_linear_stack_fwd(self.plan, self.sets[s][1].data_ptr(), self.n, self.m, stream)

    def graphs(self):
        """One CUDA graph per weight set (each = one step)."""
        torch = self.torch
        gs = []
        side = torch.cuda.Stream()
        for s in range(len(self.sets)):
            g = torch.cuda.CUDAGraph()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.graph(g, stream=side):
                self.call(s, torch.cuda.current_stream().cuda_stream)
            gs.append(g)
        torch.cuda.synchronize()
        return gs

    def check(self):
        st, bits = self.dfssm.dfssm_plan_check(self.plan)
        if st != self.dfssm.DFSSM_OK:
            raise RuntimeError(f"device error word set: {bits:#x}")

    def close(self):
        self.dfssm.dfssm_plan_destroy(self.plan)


def stack_block(torch, wl_name, seed, steps, peaks, dist, dev, weight_sets=None, layers=0):
    """One stack workload: ms per step (CUDA graph per step, two weight sets alternated), GB/s,
    tokens/s, TOPS and both roofline fractions."""
    wl = synth.WORKLOADS[wl_name]
    shapes, m, cfg = wl["shapes"], wl["m"], wl["cfg"]
    if layers:
        shapes = shapes[:2 * layers]
    r = StackRunner(shapes, m, cfg, seed, weight_sets=weight_sets)
    graphs = r.graphs()
    with ClockSampler(dev.index or 0) as clk:
        ms = timed_device(torch, lambda i: graphs[i % 2].replay(), steps, 3, dist, dev)
    r.check()
    r.close()
    del graphs
    ms_step = ms / steps
    nb, nops = stack_bytes(shapes, m), stack_ops(shapes, m)
    gbs = nb / (ms_step * 1e-3) / 1e9
    tops = nops / (ms_step * 1e-3) / 1e12
    peak_i8 = peaks["bf16"] * INT8_PER_BF16
    return {"workload": wl_name, "m": m, "steps": steps, "ms_per_step": ms_step, "GB/s": gbs,
            "tokens_per_s": m / (ms_step * 1e-3), "TOPS": tops,
            "hbm_frac": gbs / peaks["hbm"], "int8_frac": tops / peak_i8,
            "path": "decode (slice/quant + decode kernels)" if m <= 16 else "quant_rows + tcgen05 prefill",
            "clocks": clk.summary()}


def single_block(torch, wl_name, seed, peaks, dev, min_bytes=256 << 20, reps=4):
    """One projection at M = 1 with cold L2: the call rotates over enough copies of the weights
    (>= 256 MB) inside one CUDA graph; per-call latency and GB/s."""
    import bit_gemv_gemm_dfssm_b200 as dfssm
    wl = synth.WORKLOADS[wl_name]
    (d_in, d_out), m = wl["shapes"][0], wl["m"]
    w = synth.linear_weights(seed, synth.weight_cfg(wl["cfg"]), 0, d_in, d_out)
    dw = {k: torch.from_numpy(v).cuda() for k, v in w.items()}
    per = sum(v.numel() * v.element_size() for v in dw.values())
    n = (min_bytes + per - 1) // per
    copies = [{k: v.clone() for k, v in dw.items()} for _ in range(n)]
    x = torch.from_numpy(synth.activations(seed, wl["cfg"], 0, m, d_in).view(np.int16).copy()).cuda()
    y = torch.empty((m, d_out), dtype=torch.bfloat16, device="cuda")
    plan = dfssm.dfssm_linear_plan([(d_in, d_out, m, dfssm.DFSSM_BF16)])
    structs = [dfssm.weights_struct(c["sign"], c["alpha"], c["wa"], c["sa"], c["wb"], c["sb"]) for c in copies]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        st = torch.cuda.current_stream().cuda_stream
        for ws in structs:
            dfssm.dfssm_linear_fwd(plan, 0, ws, x.data_ptr(), m, y.data_ptr(), None, st)
    torch.cuda.synchronize()
    ms = timed_device(torch, lambda i: g.replay(), reps, 3, None, dev)
    st_, bits = dfssm.dfssm_plan_check(plan)
    dfssm.dfssm_plan_destroy(plan)
    del g
    if st_ != dfssm.DFSSM_OK:
        raise RuntimeError(f"device error word {bits:#x}")
    us = ms * 1e3 / (reps * n)
    nb = stack_bytes([(d_in, d_out)], m)
    return {"workload": wl_name, "m": m, "us_per_call": us, "GB/s": nb / (us * 1e-6) / 1e9,
            "hbm_frac": nb / (us * 1e-6) / 1e9 / peaks["hbm"], "tokens_per_s": m / (us * 1e-6),
            "l2": f"cold: {n} weight copies ({n * per / 2**20:.0f} MB) rotated in one CUDA graph",
            "calls_timed": reps * n}


def lm_head_block(torch, seed, peaks, dev, m=1, steps=200):
    """The int8 LM head over the tied 50,288 x 2048 table at m tokens: two tables alternated
    (2 x 103 MB > L2), one CUDA graph per call."""
    import bit_gemv_gemm_dfssm_b200 as dfssm
    vocab, d = synth.VOCAB, synth.D_MODEL
    tabs = []
    for s in range(2):
        t = synth.int8_table(seed + s, 5, vocab, d)
        tabs.append({k: torch.from_numpy(v).cuda() for k, v in t.items()})
    h = torch.from_numpy(synth.activations(seed, 5, 1, m, d).view(np.int16).copy()).cuda()
    logits = torch.empty((m, vocab), dtype=torch.bfloat16, device="cuda")
    cs = [dfssm.Int8Table(t["table"].data_ptr(), t["scale"].data_ptr(), vocab, d) for t in tabs]
    dfssm.dfssm_lm_head_fwd(cs[0], h.data_ptr(), m, logits.data_ptr(), dfssm.DFSSM_BF16, 0,
                            torch.cuda.current_stream().cuda_stream)     # the per-device set-up
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    gs = []
    for c in cs:
        side.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            dfssm.dfssm_lm_head_fwd(c, h.data_ptr(), m, logits.data_ptr(), dfssm.DFSSM_BF16, 0,
                                    torch.cuda.current_stream().cuda_stream)
        gs.append(g)
    torch.cuda.synchronize()
    ms = timed_device(torch, lambda i: gs[i % 2].replay(), steps, 3, None, dev)
    del gs
    us = ms * 1e3 / steps
    nb = vocab * d + 4 * vocab + 2 * m * d + 2 * m * vocab
    return {"workload": f"lm_head_m{m}", "vocab": vocab, "d": d, "m": m, "us_per_call": us,
            "GB/s": nb / (us * 1e-6) / 1e9, "hbm_frac": nb / (us * 1e-6) / 1e9 / peaks["hbm"],
            "bytes_per_call": nb, "l2": "two 103 MB tables alternated",
            "traffic": recorded_traffic(f"lm_head_m{m}")}


def ssm_layer_bytes(dims, m):
    """Algorithmic bytes of one layer's state step at m tokens: zxbcdt in, shift register and
    SSM state in and out, out (bf16), parameters."""
    d_inner, N, conv = dims["d_inner"], dims["d_state"], dims["d_conv"]
    nheads = d_inner // dims["headdim"]
    conv_dim = d_inner + 2 * N
    return m * (2 * (2 * d_inner + 2 * N + nheads)             # zxbcdt (bf16) in
                + 2 * 2 * conv_dim * conv                       # shift register (bf16) in and out
                + 2 * 4 * nheads * dims["headdim"] * N          # SSM state (fp32) in and out
                + 2 * d_inner) \
        + 4 * (conv_dim * conv + conv_dim + 3 * nheads + d_inner)   # parameters (fp32)


def ssm_block(torch, seed, peaks, dev, n_layers=48, m=1, steps=200):
    """The decode step of the state operations (shift register + SSM recurrence) for the 48 layers
    of Mamba-2 1.3B at m tokens: two full sets of inputs and states alternated (2 x 208 MB > L2),
    one CUDA graph per call."""
    import bit_gemv_gemm_dfssm_b200 as dfssm
    dims = synth.SSM_DIMS
    d_inner, N, conv = dims["d_inner"], dims["d_state"], dims["d_conv"]
    nheads = d_inner // dims["headdim"]
    conv_dim = d_inner + 2 * N
    c = dfssm.SsmDims(d_inner, dims["headdim"], N, conv, dims["eps"], dfssm.DFSSM_BF16)
    keep, ldevs = [], []
    for s in range(2):
        layers = []
        for i in range(n_layers):
            inp = synth.ssm_layer_inputs(seed + s, 10, i, m, dims)
            d = {k: (torch.from_numpy(v.view(np.int16).copy()) if v.dtype == np.uint16 else torch.from_numpy(v)).cuda()
                 for k, v in inp.items()}
            d["out"] = torch.empty((m, d_inner), dtype=torch.bfloat16, device="cuda")
            keep.append(d)
            layers.append(dfssm.SsmLayer(*[d[k].data_ptr() for k in ("zxbcdt", "conv_state", "ssm_state", "conv_w",
                                                                       "conv_b", "dt_bias", "a_log", "d_skip",
                                                                       "norm_w", "out")]))
        ldevs.append(torch.frombuffer(bytearray(dfssm.ssm_layers_bytes(layers)), dtype=torch.uint8).cuda())
    wsb = dfssm.dfssm_ssm_workspace_bytes(c, n_layers, m)
    ws = torch.zeros(wsb // 4 + 64, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    gs = []
    for ld in ldevs:
        side.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            dfssm.dfssm_ssm_step(c, ld.data_ptr(), n_layers, m, ws.data_ptr(), wsb, torch.cuda.current_stream().cuda_stream)
        gs.append(g)
    torch.cuda.synchronize()
    ms = timed_device(torch, lambda i: gs[i % 2].replay(), steps, 3, None, dev)
    st, bits = dfssm.dfssm_ssm_read_error(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == dfssm.DFSSM_OK, hex(bits)
    del gs
    us = ms * 1e3 / steps
    nb = n_layers * ssm_layer_bytes(dims, m)
    return {"workload": f"ssm_step{n_layers}_m{m}", "m": m, "layers": n_layers, "us_per_step": us,
            "GB/s": nb / (us * 1e-6) / 1e9, "hbm_frac": nb / (us * 1e-6) / 1e9 / peaks["hbm"],
            "bytes_per_step": nb, "tokens_per_s": m / (us * 1e-6), "gpu_launches_per_step": 2,
            "l2": "two sets of inputs and states alternated", "traffic": recorded_traffic(f"ssm_step{n_layers}_m{m}")}


def chain_bytes(n_layers, d_model, dims, vocab, m):
    """Algorithmic bytes of one chained decode step: every weight once (scaffold + LoRA + scales,
    the int8 table and its scales, the state parameters, the norm weights), the shift-register and
    SSM states in and out, and the activations between the stages (fp32 residual, bf16 between
    the kernels, fp32 logits)."""
    d_inner, N = dims["d_inner"], dims["d_state"]
    zx_w = 2 * d_inner + 2 * N + d_inner // dims["headdim"]
    lin = stack_bytes([(d_model, zx_w), (d_inner, d_model)] * n_layers, m)
    ssm = n_layers * ssm_layer_bytes(dims, m)
    d, V = d_model, vocab
    norms = (n_layers + 1) * (4 * d + m * (4 * d + 2 * d + 4 * d + 2 * d))   # w; r in, delta in, r out, out
    head = V * d + 4 * V + 2 * m * d + 4 * m * V
    embed = m * (d + 4 + 4 * d + 4)                                            # row, scale, out, id
    return lin + ssm + norms + head + embed


class ChainRunner:
    """The model's whole decode step for m tokens as one CUDA graph of the library's calls:
    the int8 embedding, then per block the residual add + RMS norm, in_proj, the state step and
    out_proj, then the last residual add + RMS norm and the int8 LM head. Every block has its own
    output buffers, so each stage's input and output can be read back after a step; the
    shift-register and SSM states are updated in place, so each replay decodes the next token."""

    def __init__(self, m, seed, n_layers=synth.N_LAYERS, d_model=synth.D_MODEL, dims=None, vocab=synth.VOCAB,
                 cfg=2):
        import torch
        import bit_gemv_gemm_dfssm_b200 as dfssm
        self.torch, self.dfssm = torch, dfssm
        dims = dict(dims or synth.SSM_DIMS)
        self.m, self.n, self.d, self.dims, self.vocab = m, n_layers, d_model, dims, vocab
        d_inner, N = dims["d_inner"], dims["d_state"]
        self.nheads = d_inner // dims["headdim"]
        self.zx_w = 2 * d_inner + 2 * N + self.nheads
        self.shapes = [(d_model, self.zx_w), (d_inner, d_model)]

        def dev(a):
            a = np.ascontiguousarray(a)
            return torch.from_numpy(a.view(np.int16).copy() if a.dtype == np.uint16 else a.copy()).cuda()

        wc = synth.weight_cfg(cfg)
        self.w_host, self.w = [], []
        for i in range(2 * n_layers):
            d_in, d_out = self.shapes[i % 2]
            w = synth.linear_weights(seed, wc, i, d_in, d_out)
            self.w_host.append(w)
            self.w.append({k: dev(v) for k, v in w.items()})
        self.ssm_host = [synth.ssm_layer_inputs(seed, cfg, i, m, dims) for i in range(n_layers)]
        self.ssm = [{k: dev(v) for k, v in x.items() if k != "zxbcdt"} for x in self.ssm_host]
        self.nw_host = [synth.block_norm_weights(seed, cfg, i, d_model) for i in range(n_layers + 1)]
        self.nw = [dev(v) for v in self.nw_host]
        self.table_host = synth.int8_table(seed, cfg, vocab, d_model)
        self.table = {k: dev(v) for k, v in self.table_host.items()}
        self.tc = dfssm.Int8Table(self.table["table"].data_ptr(), self.table["scale"].data_ptr(), vocab, d_model)
        self.ids_host = synth.token_ids(seed, cfg, m, vocab)
        self.ids = dev(self.ids_host)
        f32, bf16 = torch.float32, torch.bfloat16
        e = dict(device="cuda")
        self.emb = torch.empty((m, d_model), dtype=f32, **e)
        self.resid = [torch.empty((m, d_model), dtype=f32, **e) for _ in range(n_layers + 1)]
        self.xn = [torch.empty((m, d_model), dtype=bf16, **e) for _ in range(n_layers + 1)]
        self.zx = [torch.empty((m, self.zx_w), dtype=bf16, **e) for _ in range(n_layers)]
        self.so = [torch.empty((m, d_inner), dtype=bf16, **e) for _ in range(n_layers)]
        self.yo = [torch.empty((m, d_model), dtype=bf16, **e) for _ in range(n_layers)]
        self.logits = torch.empty((m, vocab), dtype=f32, **e)
        self.plan = dfssm.dfssm_linear_plan([(d_in, d_out, m, dfssm.DFSSM_BF16) for d_in, d_out in self.shapes])
        self.c = dfssm.SsmDims(d_inner, dims["headdim"], N, dims["d_conv"], dims["eps"], dfssm.DFSSM_BF16)
        layers = [dfssm.SsmLayer(self.zx[i].data_ptr(), *[self.ssm[i][k].data_ptr() for k in (
            "conv_state", "ssm_state", "conv_w", "conv_b", "dt_bias", "a_log", "d_skip", "norm_w")],
            self.so[i].data_ptr()) for i in range(n_layers)]
        self.layer_bytes = len(dfssm.ssm_layers_bytes(layers[:1]))
        self.ldev = torch.frombuffer(bytearray(dfssm.ssm_layers_bytes(layers)), dtype=torch.uint8).cuda()
        self.wsb = dfssm.dfssm_ssm_workspace_bytes(self.c, 1, m)
        self.ws = torch.zeros(self.wsb // 4 + 64, dtype=torch.int32, **e)
        self.ws_ptr = (self.ws.data_ptr() + 255) // 256 * 256
        self.ws_ptr_bytes = self.wsb
        # the per-device set-up of the table calls, before any capture
        stream = torch.cuda.current_stream().cuda_stream
        dfssm.dfssm_embed_fwd(self.tc, self.ids.data_ptr(), m, self.emb.data_ptr(), dfssm.DFSSM_F32, 0, stream)
        torch.cuda.synchronize()

    def weights(self, i):
        w = self.w[i]
        return self.dfssm.weights_struct(w["sign"], w["alpha"], w["wa"], w["sa"], w["wb"], w["sb"])

    def step(self, stream):
        """Enqueue one decode step (1 + 7 n + 2 kernel launches)."""
        dfssm, m, d = self.dfssm, self.m, self.d
        BF16, F32 = dfssm.DFSSM_BF16, dfssm.DFSSM_F32
        eps = self.dims["eps"]
        dfssm.dfssm_embed_fwd(self.tc, self.ids.data_ptr(), m, self.emb.data_ptr(), F32, 0, stream)
        for i in range(self.n):
            r_in = self.emb if i == 0 else self.resid[i - 1]
            delta = 0 if i == 0 else self.yo[i - 1].data_ptr()
            dfssm.dfssm_add_rmsnorm(self.nw[i].data_ptr(), d, eps, r_in.data_ptr(), delta, BF16, m,
                                    self.resid[i].data_ptr(), self.xn[i].data_ptr(), BF16, stream)
            dfssm.dfssm_linear_fwd(self.plan, 0, self.weights(2 * i), self.xn[i].data_ptr(), m, self.zx[i].data_ptr(),
                                   None, stream)
            dfssm.dfssm_ssm_step(self.c, self.ldev.data_ptr() + i * self.layer_bytes, 1, m, self.ws_ptr,
                                 self.ws_ptr_bytes, stream)
            dfssm.dfssm_linear_fwd(self.plan, 1, self.weights(2 * i + 1), self.so[i].data_ptr(), m,
                                   self.yo[i].data_ptr(), None, stream)
        n = self.n
        dfssm.dfssm_add_rmsnorm(self.nw[n].data_ptr(), d, eps, self.resid[n - 1].data_ptr(), self.yo[n - 1].data_ptr(),
                                BF16, m, self.resid[n].data_ptr(), self.xn[n].data_ptr(), BF16, stream)
        dfssm.dfssm_lm_head_fwd(self.tc, self.xn[n].data_ptr(), m, self.logits.data_ptr(), F32, 0, stream)

    def launches(self):
        return 1 + 7 * self.n + 2

    def graph(self):
        torch = self.torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self.step(torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        return g

    def bytes_per_step(self):
        return chain_bytes(self.n, self.d, self.dims, self.vocab, self.m)

    def check(self):
        st, bits = self.dfssm.dfssm_ssm_read_error(self.ws_ptr, self.torch.cuda.current_stream().cuda_stream)
        if st != self.dfssm.DFSSM_OK:
            raise RuntimeError(f"state step error word set: {bits:#x}")
        st, bits = self.dfssm.dfssm_plan_check(self.plan)
        if st != self.dfssm.DFSSM_OK:
            raise RuntimeError(f"linear error word set: {bits:#x}")

    def close(self):
        self.dfssm.dfssm_plan_destroy(self.plan)


def chain_block(torch, seed, peaks, dev, m=1, steps=100):
    """The model's whole decode step (48 blocks of Mamba-2 1.3B with the layer in every in_proj
    and out_proj, embedding and LM head in int8) at m tokens, one CUDA graph per step; each step
    decodes the next token (the states carry over). Reads about 480 MB per token, well above L2."""
    r = ChainRunner(m, seed)
    g = r.graph()
    ms = timed_device(torch, lambda i: g.replay(), steps, 3, None, dev)
    r.check()
    del g
    r.close()
    us = ms * 1e3 / steps
    nb = r.bytes_per_step()
    return {"workload": f"decode_step48_m{m}", "m": m, "layers": r.n, "us_per_step": us,
            "tokens_per_s": m / (us * 1e-6), "GB/s": nb / (us * 1e-6) / 1e9,
            "hbm_frac": nb / (us * 1e-6) / 1e9 / peaks["hbm"], "bytes_per_step": nb,
            "gpu_launches_per_step": r.launches(), "l2": "one step reads every weight and state once (~480 MB)"}


def timed_device(torch, run_step, steps, warmup, dist, dev):
    for i in range(warmup):
        run_step(i)
    torch.cuda.synchronize()
    if dist is not None and dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        run_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None and dist.is_initialized():
        dist.barrier()
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, dist, dev)


def run_gpu(args, wl_name):
    import torch
    ws, rank, local = dist_env()
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist_mod
        dist = dist_mod
        backend = os.environ.get("DFSSM_BENCH_BACKEND", "nccl")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    wl = synth.WORKLOADS[wl_name]
    shapes, m, cfg = wl["shapes"], wl["m"], wl["cfg"]
    if args.layers:
        shapes = shapes[:2 * args.layers]
    seed = replica_seed(rank)

    r = StackRunner(shapes, m, cfg, seed)
    graphs = r.graphs()
    nb = stack_bytes(shapes, m)
    nops = stack_ops(shapes, m)

    def step(i):
        graphs[i % 2].replay()

    with ClockSampler(local) as clk:
        ms = timed_device(torch, step, args.steps, args.warmup, dist, dev)
    r.check()
    ms_step = ms / args.steps
    total_units = sum_over_ranks(float(m * args.steps), dist, dev)      # tokens, all ranks
    total_bytes = sum_over_ranks(float(nb * args.steps), dist, dev)
    value_gbs = total_bytes / (ms * 1e-3) / 1e9
    tok_s = total_units / (ms * 1e-3)
    achieved = nb / (ms_step * 1e-3) / 1e9

    # end to end through the C ABI with host buffers, every step: pinned host x -> device (one
    # copy), then the stack call with each entry's y in pinned host memory, which the kernels
    # write over PCIe as they finish each row (the device -> host transfer overlaps the compute).
    e2e = None
    if not args.no_e2e:
        y_host_dev = mapped_address(r.y_host.data_ptr())
        host_sets = [r.entries(ws, y_host_dev) for ws, _ in r.sets]
        stream = torch.cuda.current_stream()

        def e2e_step(i):
            r.x.copy_(r.x_host, non_blocking=True)
            r.dfssm.dfssm_linear_stack_fwd(r.plan, host_sets[i % 2].data_ptr(), r.n, r.m, stream.cuda_stream)

        e2e_ms = timed_device(torch, e2e_step, args.steps, args.warmup, dist, dev)
        # the host outputs equal those of the same call writing device memory
        last = r.y_host.clone()
        r.call((args.steps - 1) % 2, stream.cuda_stream)
        torch.cuda.synchronize()
        if not torch.equal(r.y.view(torch.int16).cpu(), last):
            raise RuntimeError("outputs written to host memory differ from those written to device memory")
        e2e = {"value": sum_over_ranks(float(nb * args.steps), dist, dev) / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "ms_per_step": e2e_ms / args.steps, "h2d_bytes_per_step": r.x_elems * 2,
               "d2h_bytes_per_step": r.y_elems * 2, "y": "pinned host memory, written by the kernels"}
    r.check()
    r.close()
    del graphs

    # prefill pass (M = 2048): int8 tensor-core TOPS
    prefill = None
    if not args.no_prefill:
        pwl = synth.WORKLOADS["stack48_m2048"]
        pshapes = pwl["shapes"][:2 * args.layers] if args.layers else pwl["shapes"]
        pr = StackRunner(pshapes, pwl["m"], pwl["cfg"], seed)
        psteps = args.prefill_steps
        pgraphs = pr.graphs()
        with ClockSampler(local) as pclk:
            pms = timed_device(torch, lambda i: pgraphs[i % 2].replay(), psteps, max(3, args.warmup // 10), dist, dev)
        pr.check()
        pops = stack_ops(pshapes, pwl["m"])
        tops = sum_over_ranks(float(pops * psteps), dist, dev) / (pms * 1e-3) / 1e12
        peak_i8 = peaks["bf16"] * INT8_PER_BF16
        ach = pops / (pms / psteps * 1e-3) / 1e12
        prefill = {
            "workload": "stack48_m2048", "m": pwl["m"], "steps": psteps, "ms_per_step": pms / psteps,
            "value": tops, "unit": "TOPS", "tokens_per_s": sum_over_ranks(float(pwl["m"] * psteps), dist, dev)
            / (pms * 1e-3),
            "roofline": {"bound": "tensor", "achieved": ach, "peak": peak_i8, "unit": "TOPS",
                         "frac": ach / peak_i8, "traffic": recorded_traffic("stack48_m2048"),
                         "peak_source": f"int8 = {INT8_PER_BF16:g} x {peaks['src']} bf16 burst"},
            "clocks": pclk.summary(),
        }
        pr.close()
        del pgraphs

    # the other configurations: single projections (cold L2), the stack at M = 4 / 16 / 64 / 512,
    # the int8 LM head, the decode step of the state operations, the model's whole chained decode
    # step (every rank runs the same blocks; rank 0 reports them)
    extras = None
    if not args.no_extras:
        extras = {"single": [], "stacks": [], "lm_head": None, "ssm_step": None, "decode_step": None}
        for wn in ("out_proj_m1", "in_proj_m1"):
            extras["single"].append(single_block(torch, wn, seed, peaks, dev))
        sets = device_weight_sets(synth.stack_shapes(), 2, seed)
        for wn, st in (("stack48_m4", 300), ("stack48_m16", 200), ("stack48_m64", 100), ("stack48_m512", 20)):
            extras["stacks"].append(stack_block(torch, wn, seed, st, peaks, dist, dev, weight_sets=sets))
        del sets
        torch.cuda.empty_cache()
        extras["lm_head"] = lm_head_block(torch, seed, peaks, dev)
        torch.cuda.empty_cache()
        extras["ssm_step"] = ssm_block(torch, seed, peaks, dev)
        torch.cuda.empty_cache()
        extras["decode_step"] = chain_block(torch, seed, peaks, dev)

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    cpu = None
    if ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_leg(shapes, m, seed, cfg)

    line = {
        "metric": metric_name(), "value": value_gbs, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 x 1-bit -> int32, fp32 epilogue, bf16 out",
        "data": "synthetic (seeded; Mamba-2-1.3B shapes, random weights)",
        "config": {"workload": wl_name if not args.layers else f"{wl_name} (first {args.layers} layers)",
                   "m": m, "linears": len(shapes), "layers": len(shapes) // 2,
                   "d_model": 2048, "rank": 16, "parallelism": f"replicas x{ws}",
                   "l2": "two weight sets alternated per step (2 x 171.8 MB > 126 MB L2)",
                   "bytes_per_step": nb, "graph": "one CUDA graph per step"},
        "tokens_per_s": tok_s,
        "tops": sum_over_ranks(float(nops * args.steps), dist, dev) / (ms * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm"], "traffic": recorded_traffic(wl_name),
                     "peak_source": f"{peaks['src']} copy bandwidth",
                     "timed": ("lora_slice_kernel + decode_kernel" if m == 1 else
                               "quant_kernel + decode_kernel" if m <= 16 else "quant_rows_kernel + prefill_kernel")
                     + " per call (PDL-overlapped)"},
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
        "prefill": prefill,
        "workloads": extras,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="dfssm", choices=["dfssm", "reference"])
    ap.add_argument("--workload", default="stack48_m1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--prefill-steps", type=int, default=30)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations (single projections, M = 4/16/64/512, LM head)")
    ap.add_argument("--layers", type=int, default=0,
                    help="use only the first L layers of the stack (small cases for profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args, args.workload)
    return run_gpu(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
