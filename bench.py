"""FAVOR+ benchmark: tokens/s (B*H*L) of one pass of the hot path, and its roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2|3|4|5] [--impl ours|reference]

A step is one pass of the whole hot path (every kernel favor_fwd launches, plus favor_bwd for the
forward+backward workload) over one batch of seeded synthetic input already resident in HBM.
Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device synchronise;
each step is timed with CUDA events on the launching stream and the L2 cache is flushed (a
256 MB write) between steps outside the timed events; the job time is the max over ranks. One
JSON line is printed by rank 0. Under torchrun each rank runs its own replica of the workload
(independent heads; weak scaling, no data-path collective).

--impl reference times the fp64 oracle (the method's plain CPU definition) on the host cores on a
bounded sample of the same workload; under torchrun only rank 0 runs it.
"""

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_positive_b200.inputs import WORKLOADS, make_inputs, round_to_bf16  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TF32_PER_BF16 = 1.1 / 2.25   # nominal dense tf32 : bf16 tensor rate
L2_FLUSH_BYTES = 256 << 20

# Kernels favor_fwd launches for the bf16 path, in launch order (stage k <-> events 2k, 2k+1); for
# d = 64 the key-state kernel is k_key_partials_wide (128-token key tiles).
FWD_STAGES = ["k_key_partials", "k_state_image", "k_query_out"]
CAUSAL_STAGES = ["k_key_partials_wide", "k_segment_scan", "k_causal_chunk", "gemm_causal_prefix"]
# Kernels favor_bwd launches (bf16 bidirectional: split-precision GEMM passes and two reductions).
BWD_STAGES = ["gemm_phi_k", "gemm_state_partial", "reduce_state", "gemm_phi_q", "gemm_gs", "gemm_t_q", "gemm_dq",
              "gemm_G_partial", "reduce_G", "gemm_dv", "gemm_t_k", "gemm_dk"]
# (bf16 causal: the same passes split at 128-token chunks, with masked diagonal tiles and
# per-chunk prefix / suffix state images)
BWD_CAUSAL_STAGES = ["gemm_phi_k", "gemm_phi_q", "gemm_chunk_state", "scan_prefix", "gemm_mask_A", "gemm_nd_inter",
                     "gemm_gs_intra", "gemm_mask_B", "gemm_dphiq_inter", "gemm_t_q_intra", "gemm_dq", "gemm_chunk_G",
                     "scan_suffix", "gemm_dv_inter", "gemm_dv_intra", "gemm_dphik_inter", "gemm_t_k_intra", "gemm_dk"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def stage_work(name, w, n_sms=148):
    """Algorithmic HBM bytes and tensor FLOPs (bf16/fp16 rate, tf32 rate) of one launch of a stage."""
    t, d, m = w.tokens, w.d, w.m
    BH = w.B * w.H
    if name in ("k_key_partials", "k_key_partials_wide"):  # read K, V; MMAs K W^T and phi'(K)^T [V | 1]
        if w.causal:                   # the causal instantiation also writes -|k|^2/2 per key
            return t * (4 * d + 4), 2 * m * d * t + 2 * m * (d + 1) * t, 0
        return t * 4 * d, 2 * m * d * t + 2 * m * (d + 1) * t, 0
    if name == "k_state_image":        # read the per-run partial states and stabilisers, write the fp16 images
        runs = n_sms + BH - 1
        return runs * (d + 2) * m * 4 + BH * (d // 64) * (m // 128) * 20480, 0, 0
    if name == "k_segment_scan":       # read the per-segment states and stabilisers, write the prefixes
        n_seg = BH * ((((w.L + 127) // 128) + 7) // 8)
        return n_seg * m * (2 * (d + 1) + 1) * 4, 0, 0
    if name == "k_query_out":          # read Q; write fp32 out; MMAs Q W^T and phi(Q) [S | z]
        return t * (2 * d + 4 * d), 2 * m * d * t + 2 * m * (d + 1) * t, 0
    # Backward passes: the bytes each launch must move given the materialised hi/lo bf16
    # intermediates (4 B per element: phi(K), phi(Q), t are m wide, [g | s] is d + 64 wide) and the
    # tensor FLOPs of its split products (3 MMAs when both operands are split, 2 when one is exact).
    Np = d + 64
    mf = 2 * m if w.feature_map == "trig" else m   # features per token (sin and cos: 2m)
    if name in ("gemm_phi_k", "gemm_phi_q"):   # read K (or Q); write phi hi/lo
        return t * (2 * d + 4 * mf), 2 * m * d * t, 0
    if name == "gemm_state_partial":           # read phi(K) hi/lo and V
        return t * (4 * mf + 2 * d), 2 * 2 * mf * (d + 1) * t, 0
    if name == "sp_state+sp_output":           # both calls: read K, V, Q; phi hi/lo out and back; out
        return t * (6 * d + 2 * 8 * m + 4 * d), (2 * 2 * m * d + 2 * 2 * m * (d + 1) + 3 * 2 * m * (d + 1)) * t, 0
    if name == "gemm_out":                     # read phi(Q) hi/lo; write fp32 out
        return t * (4 * mf + 4 * d), 3 * 2 * mf * (d + 1) * t, 0
    if name == "gemm_G_partial":               # read phi(Q) hi/lo and [g | s] hi/lo
        return t * (4 * m + 4 * Np), 3 * 2 * m * (d + 1) * t, 0
    if name in ("reduce_state", "reduce_G"):   # read the partial states, write the hi/lo images
        return 0, 0, 0
    if name == "gemm_gs":                      # read phi(Q) hi/lo and dO; write [g | s] hi/lo
        return t * (4 * m + 2 * d + 4 * Np), 3 * 2 * m * (d + 1) * t, 0
    if name == "gemm_t_q":                     # read [g | s] and phi(Q) hi/lo; write t hi/lo and sum t
        return t * (4 * Np + 8 * m + 4), 3 * 2 * m * (d + 1) * t, 0
    if name in ("gemm_dq", "gemm_dk"):         # read t hi/lo, x and sum t; write dx fp32
        return t * (4 * m + 2 * d + 4 + 4 * d), 2 * 2 * m * d * t, 0
    if name == "gemm_dv":                      # read phi(K) hi/lo; write dV fp32
        return t * (4 * m + 4 * d), 3 * 2 * m * d * t, 0
    if name == "gemm_t_k":                     # read V and phi(K) hi/lo; write t hi/lo and sum t
        return t * (2 * d + 8 * m + 4), 2 * 2 * m * (d + 1) * t, 0
    C = 128  # causal backward chunk
    if name == "gemm_chunk_state":             # read phi(K) hi/lo and V
        return t * (4 * m + 2 * d), 2 * 2 * m * (d + 1) * t, 0
    if name == "gemm_chunk_G":                 # read phi(Q) hi/lo and [g | s] hi/lo
        return t * (4 * m + 4 * Np), 3 * 2 * m * (d + 1) * t, 0
    if name in ("scan_prefix", "scan_suffix"):
        return 0, 0, 0
    if name == "gemm_mask_A":                  # read phi(Q), phi(K) hi/lo; write the masked tile hi/lo
        return t * (8 * m + 4 * C), 3 * 2 * m * C * t, 0
    if name == "gemm_nd_inter":                # read phi(Q) hi/lo; write fp32 [num | den] part
        return t * (4 * m + 4 * Np), 3 * 2 * m * (d + 1) * t, 0
    if name == "gemm_gs_intra":                # read A, V, the fp32 part and dO; write [g | s] hi/lo
        return t * (4 * C + 4 * d + 8 * Np), 2 * 2 * C * (d + 1) * t, 0
    if name == "gemm_mask_B":                  # read [g | s] hi/lo and V; write the masked tile hi/lo
        return t * (4 * Np + 2 * d + 4 * C), 2 * 2 * C * (d + 1) * t, 0
    if name == "gemm_dphiq_inter":             # read [g | s] hi/lo; write fp32 part
        return t * (4 * Np + 4 * m), 3 * 2 * m * (d + 1) * t, 0
    if name in ("gemm_t_q_intra", "gemm_t_k_intra"):  # read B, phi (two), the part; write t hi/lo
        return t * (4 * C + 12 * m + 4 * m + 4), 3 * 2 * C * m * t, 0
    if name == "gemm_dv_inter":                # read phi(K) hi/lo; write fp32 part
        return t * (4 * m + 4 * d), 3 * 2 * m * d * t, 0
    if name == "gemm_dv_intra":                # read A, g hi/lo and the part; write dV
        return t * (4 * C + 4 * d + 8 * d), 3 * 2 * C * d * t, 0
    if name == "gemm_dphik_inter":             # read V; write fp32 part
        return t * (2 * d + 4 * m), 2 * 2 * m * (d + 1) * t, 0
    if name == "gemm_causal_prefix":   # first 512 tokens per head at split precision (four GEMMs):
        # read q, k, v; write and read phi hi/lo and the masked scores hi/lo; write out
        P = min(w.L, 512)
        Pp = (P + 127) // 128 * 128
        nbytes = BH * P * (6 * d + 2 * 8 * m + 2 * 4 * Pp + 4 * d)
        flops = BH * P * (2 * 2 * m * d + 3 * 2 * m * Pp + 2 * 2 * Pp * (d + 1))
        return nbytes, flops, 0
    if name == "k_causal_chunk":       # read Q, K, V, -|k|^2/2; write fp32 out; fp16 MMAs per token:
        # Q W^T and K W^T (2 x 2md), state term and state update (2 x 2md), scores and masked A V
        # over the 128-token tile (2 * 128 * m + 2 * 128 * d)
        return t * (10 * d + 4), (8 * m * d + 2 * 128 * m + 2 * 128 * d) * t, 0
    return 0, 0, 0


def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_positive_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel, workload_name):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_sha") != source_hash() or rec.get("workload") != workload_name:
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every ~0.5 ms through NVML while the timed
    region runs (a background thread; the timed steps themselves take a few milliseconds)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, device):
        self.device = device
        self.samples = []
        self.thread = None
        self.stop_flag = threading.Event()

    def _handle(self, pynvml):
        try:
            p = torch.cuda.get_device_properties(self.device)
            bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device)

    def _run(self, pynvml, h):
        while not self.stop_flag.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, rs))
            except Exception:
                return
            time.sleep(0.0005)

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
        except Exception:
            return
        self.thread = threading.Thread(target=self._run, args=(pynvml, h), daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        sm = [a for a, _, _ in self.samples]
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        reasons = sorted({name for _, _, r in self.samples for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(m for _, m, _ in self.samples),
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------------------------------ oracle arm

def oracle_sample(w, x, W64, heads):
    """Runs the fp64 oracle over ``heads`` (b, h) pairs of the workload; returns tokens done."""
    from oracle import favor

    for b, h in heads:
        X = {k: x[k][b, h].astype(np.float64) for k in x}
        if w.backward:
            favor.fwd(X["Q"][None, None], X["K"][None, None], X["V"][None, None], W64, causal=w.causal)
            favor.bwd(X["Q"][None, None], X["K"][None, None], X["V"][None, None], W64, X["dO"][None, None],
                      causal=w.causal)
        else:
            favor.fwd(X["Q"][None, None], X["K"][None, None], X["V"][None, None], W64, causal=w.causal)
    return len(heads) * w.L


def pick_sample(w, x, W64, budget_s):
    """Number of heads whose oracle run takes about budget_s seconds (at least one)."""
    t0 = time.perf_counter()
    oracle_sample(w, x, W64, [(0, 0)])
    per_head = time.perf_counter() - t0
    return max(1, min(w.B * w.H, int(budget_s / max(per_head, 1e-6))))


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = make_inputs(w)
    W64 = oracle_W(w)
    n_heads = pick_sample(w, x, W64, budget_s=max(1.0, 60.0 / max(args.steps + args.warmup, 1)))
    heads = [(i // w.H, i % w.H) for i in range(n_heads)]
    for _ in range(args.warmup):
        oracle_sample(w, x, W64, heads[:1])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        toks = oracle_sample(w, x, W64, heads)
        times.append(time.perf_counter() - t0)
    sec = statistics.mean(times)
    value = toks / sec
    sample = f"{n_heads} of {w.B * w.H} heads (L={w.L}) per step, fp64 numpy oracle"
    line = {
        "impl": "reference", "metric": metric_name(w), "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def api_draw(w):
    from linear_attention_positive_b200 import api

    return api.draw_features(w.w_seed, w.m, w.d)


def oracle_W(w):
    """W as the oracle consumes it: the oracle's own draw, rounded to the workload's dtype (the
    same values the kernels read; the library's draw is pinned bit-identical to it)."""
    from oracle import features

    W = features.draw_W(w.w_seed, w.m, w.d).astype(np.float32)
    return (round_to_bf16(W) if w.dtype == "bf16" else W).astype(np.float64)


def metric_name(w):
    kind = "fwd+bwd" if w.backward else "fwd"
    if w.feature_map != "positive":
        return f"{w.feature_map}-feature attention {kind} tokens/s (B*H*L)"
    return f"FAVOR+ {kind} tokens/s (B*H*L)"


def workload_config(w, n):
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "m": w.m, "causal": w.causal,
            "backward": w.backward, "global_batch": w.B * n, "seq_len": w.L, "parallelism": f"replicas{n}",
            "l2": "flushed between steps (256 MB write, outside the timed events)"}


# ------------------------------------------------------------------------------------ ranks

def max_over_ranks(values, world, device=None):
    """Element-wise maximum of a list of floats over all ranks (one all-reduce MAX; the job takes as
    long as its slowest rank). At world size 1 the values come back unchanged."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_rate(tokens_per_rank, world, job_ms, steps):
    """(ms per step, whole-job tokens/s) for `steps` steps that took job_ms on the slowest rank, each
    rank processing tokens_per_rank per step (weak scaling: the per-rank work is fixed)."""
    ms_per_step = job_ms / steps
    return ms_per_step, tokens_per_rank * world / (ms_per_step * 1e-3)


# ------------------------------------------------------------------------------------ GPU arm

MAP_STAGES = ["gemm_phi_k", "gemm_state_partial", "reduce_state", "gemm_phi_q", "gemm_out"]
# the sequence-parallel calls, timed as one step (no per-launch events)
SP_STAGES = ["sp_state", "sp_output"]
MAP_CODES = {"positive": 0, "relu": 1, "trig": 2}


def stage_names(w):
    """Kernel launches of one step, in launch order (stage k <-> stage events 2k, 2k+1); the
    backward's launches follow the forward's."""
    if w.feature_map != "positive":
        return list(MAP_STAGES)
    if w.sequence_parallel:
        return list(SP_STAGES)
    if w.dtype != "bf16":
        return ["k_f32_head"] + (["k_f32_head_bwd"] if w.backward else [])
    names = list(CAUSAL_STAGES if w.causal else FWD_STAGES)
    if not w.causal and w.d == 64:
        names[0] = "k_key_partials_wide"
    if w.backward:
        names += BWD_CAUSAL_STAGES if w.causal else BWD_STAGES
    return names


def stage_exps(name, w):
    """MUFU transcendental evaluations (exp2; sin and cos for the trigonometric map) of one launch."""
    t, m = w.tokens, w.m
    per_feature = 0 if w.feature_map == "relu" else (2 if w.feature_map == "trig" else 1)
    if name in ("k_key_partials", "k_key_partials_wide", "k_query_out", "gemm_phi_k",
                "gemm_phi_q"):
        return per_feature * m * t
    if name in ("k_causal_chunk", "sp_state+sp_output"):
        return 2 * per_feature * m * t
    return 0


def stage_roofline(name, w, ms, peaks, peak_src, n_sms, clk=None, traffic_key=None):
    """The launch against the slowest of its three bounds: HBM bytes at the copy bandwidth, tensor
    FLOPs at the bf16 rate, and MUFU exponentials at 16 per clock per SM at the sampled SM clock
    (reported as "alu": the special-function unit is the arithmetic unit that binds)."""
    nbytes, f_bf16, f_tf32 = stage_work(name, w, n_sms)
    exps = stage_exps(name, w)
    sec = ms * 1e-3
    hbm_peak, tc_peak = peaks["hbm_gbs"], peaks["bf16_tflops"]
    mhz = clk["sm_mhz"] if clk and clk.get("sm_mhz") else 1965.0
    mufu_peak = 16 * n_sms * mhz * 1e6 / 1e9   # G ex2 / s
    t_hbm = nbytes / (hbm_peak * 1e9)
    t_tc = f_bf16 / (tc_peak * 1e12) + f_tf32 / (tc_peak * TF32_PER_BF16 * 1e12)
    t_mufu = exps / (mufu_peak * 1e9)
    traffic = measured_traffic(name, traffic_key or w.name)
    if t_mufu > max(t_tc, t_hbm):
        return {"kernel": name, "bound": "alu", "achieved": exps / sec / 1e9, "peak": mufu_peak, "unit": "Gexp2/s",
                "frac": (exps / sec / 1e9) / mufu_peak, "traffic": traffic, "algorithmic_exps": exps,
                "note": f"MUFU ex2 at 16 per clock per SM x {n_sms} SMs at {mhz:.0f} MHz; the tensor bound "
                        f"({t_tc * 1e6:.1f} us) and the HBM bound ({t_hbm * 1e6:.1f} us, {peak_src} copy "
                        f"bandwidth) are lower"}
    if t_tc > t_hbm:
        eq = f_bf16 + f_tf32 / TF32_PER_BF16
        return {"kernel": name, "bound": "tensor", "achieved": eq / sec / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": (eq / sec / 1e12) / tc_peak, "traffic": traffic, "algorithmic_flops": eq,
                "note": f"bf16-equivalent FLOPs per launch (tf32 at the nominal {TF32_PER_BF16:.3f}x rate); "
                        f"peak {peak_src} burst bf16"}
    return {"kernel": name, "bound": "hbm", "achieved": nbytes / sec / 1e9, "peak": hbm_peak, "unit": "GB/s",
            "frac": (nbytes / sec / 1e9) / hbm_peak, "traffic": traffic, "algorithmic_bytes": nbytes,
            "note": f"peak {peak_src} copy bandwidth"}


def path_roofline(w, ms_per_step, peaks, clk, n_sm):
    """Path-level fractions (work of the definition, not of the kernels): Q, K, V (and dO) bf16 read,
    out (and dQ, dK, dV) fp32 written, at the copy bandwidth; 6 L m d FLOPs per head for the
    forward (twice that again for the backward) at the bf16 rate; 2 m exponentials per
    token per pass at 16 MUFU ex2 per clock per SM, at the SM clock sampled during the timed steps."""
    bwd = 1 if w.backward else 0
    path_bytes = w.tokens * ((6 * w.d + 4 * w.d) + bwd * (8 * w.d + 12 * w.d))
    path_flops = (6 + 12 * bwd) * w.tokens * w.m * w.d
    # transcendental evaluations: exp (positive map), sin and cos (trigonometric); none for ReLU
    path_exps = 0 if w.feature_map == "relu" else (2 + 2 * bwd) * w.m * w.tokens
    step_s = ms_per_step * 1e-3
    sm_hz = (clk["sm_mhz"] if clk and clk.get("sm_mhz") else 1965.0) * 1e6
    return {"hbm_bytes_per_step": path_bytes, "hbm_frac": path_bytes / step_s / (peaks["hbm_gbs"] * 1e9),
            "tensor_flops_per_step": path_flops, "tensor_frac": path_flops / step_s / (peaks["bf16_tflops"] * 1e12),
            "exps_per_step": path_exps, "mufu_frac": path_exps / step_s / (16 * n_sm * sm_hz),
            "note": "hbm: bf16 inputs + fp32 outputs at the copy bandwidth; tensor: 6 L m d per head forward, "
                    "12 L m d backward, at the bf16 peak (peaks: MEASURED_PEAKS.json when present, else the "
                    "fallback); mufu: 2 m ex2 per token per pass at 16 per clock per SM"}


class Runner:
    """One workload resident on the device, timed step by step with CUDA events."""

    def __init__(self, w, dev, api, torch, exp_poly_pct=0):
        self.w, self.dev, self.api, self.torch = w, dev, api, torch
        self.x = make_inputs(w)
        Wf = api_draw(w).astype(np.float32)
        self.tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.T = {k: torch.from_numpy(self.x[k]).to(self.tdt).to(dev) for k in self.x}
        self.Wt = torch.from_numpy(round_to_bf16(Wf) if w.dtype == "bf16" else Wf).to(self.tdt).to(dev)
        shape = api.make_shape(w.B, w.H, w.L, w.d, w.m, api.FAVOR_BF16 if w.dtype == "bf16" else api.FAVOR_F32)
        mo = api.make_opts(feature_map=MAP_CODES[w.feature_map])
        self.ws = torch.empty(max(api.workspace_size(shape, w.causal, False, mo),
                                  api.workspace_size(shape, w.causal, w.backward, mo)),
                              dtype=torch.uint8, device=dev)
        self.ctx = torch.empty(api.ctx_size(shape, w.causal), dtype=torch.uint8, device=dev) if w.backward else None
        self.out = torch.empty(self.T["Q"].shape, dtype=torch.float32, device=dev)
        self.grads = [torch.empty(self.T["Q"].shape, dtype=torch.float32, device=dev) for _ in range(3)] \
            if w.backward else None
        if w.sequence_parallel:
            self.sp_state = torch.empty(api.library().favor_sp_state_size(api.ctypes.byref(shape)) // 4,
                                        dtype=torch.float32, device=dev)
            self.sp_ws = torch.empty(api.library().favor_sp_workspace_size(api.ctypes.byref(shape)),
                                     dtype=torch.uint8, device=dev)
        self.stages = stage_names(w)
        self.poly = exp_poly_pct
        self.fmap = MAP_CODES[w.feature_map]
        self.base_opts = api.make_opts(exp_poly_pct=exp_poly_pct, feature_map=self.fmap)

    def step(self, T=None, fwd_opts=None, bwd_opts=None, outs=None):
        """One pass of the path on the current stream; ``outs`` = [out (, dQ, dK, dV)] to write into
        other buffers than the runner's own."""
        api, w = self.api, self.w
        T = T or self.T
        out, grads = (outs[0], outs[1:]) if outs else (self.out, self.grads)
        if w.sequence_parallel:
            # one rank's two calls; a multi-GPU run adds the all-reduce of the state in between
            api.sp_state(T["K"], T["V"], self.Wt, state=self.sp_state, workspace=self.sp_ws)
            api.sp_output(T["Q"], self.Wt, self.sp_state, out=out, workspace=self.sp_ws)
            return
        api.fwd(T["Q"], T["K"], T["V"], self.Wt, causal=w.causal, out=out, ctx=self.ctx, workspace=self.ws,
                opts=fwd_opts or self.base_opts)
        if w.backward:
            api.bwd_into(T["Q"], T["K"], T["V"], self.Wt, out, T["dO"], *grads, ctx=self.ctx,
                         causal=w.causal, workspace=self.ws, opts=bwd_opts)

    def n_fwd_stages(self):
        return len(self.stages) - (len(BWD_CAUSAL_STAGES if self.w.causal else BWD_STAGES)
                                   if self.w.backward and self.w.dtype == "bf16" else 0)

    def time(self, steps, warmup, flush, world, dist):
        torch, api = self.torch, self.api
        stream = torch.cuda.current_stream()

        def new_events(n):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            for e in evs:
                e.record()
            return evs

        for _ in range(warmup):
            flush.zero_()
            self.step()
        torch.cuda.synchronize()
        if api.sync_status() != api.FAVOR_OK:
            raise RuntimeError(f"device status not OK after warm-up ({self.w.name})")
        # timed steps: events around each whole step only (an event recorded between two launches
        # would keep the second from starting its prologue under the first's tail)
        step_ev = [new_events(2) for _ in range(steps)]
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for k in range(steps):
            flush.zero_()
            step_ev[k][0].record(stream)
            self.step()
            step_ev[k][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        status = api.sync_status()
        step_ms = [a.elapsed_time(b) for a, b in step_ev]
        # per-kernel breakdown from further steps with an event pair around every launch
        fev = [new_events(2 * api.FAVOR_MAX_STAGES) for _ in range(steps)]
        bev = [new_events(2 * api.FAVOR_MAX_STAGES) for _ in range(steps)]
        fopts = [api.make_opts(exp_poly_pct=self.poly, stage_events=fev[k], feature_map=self.fmap)
                 for k in range(steps)]
        bopts = [api.make_opts(stage_events=bev[k]) for k in range(steps)]
        torch.cuda.synchronize()
        for k in range(steps):
            flush.zero_()
            self.step(fwd_opts=fopts[k], bwd_opts=bopts[k])
        torch.cuda.synchronize()
        nf = self.n_fwd_stages()
        stage_ms = {}
        if self.w.sequence_parallel:  # the two calls record no per-launch events
            return step_ms, {"sp_state+sp_output": statistics.mean(step_ms)}, status
        for i, name in enumerate(self.stages):
            ev, j = (fev, i) if i < nf else (bev, i - nf)
            key = name if name not in stage_ms else f"{name}#{i}"
            stage_ms[key] = statistics.mean(ev[k][2 * j].elapsed_time(ev[k][2 * j + 1]) for k in range(steps))
        return step_ms, stage_ms, status

    def e2e(self, steps, flush, world, dist):
        """Through the public API: every step, the inputs come in from pinned host memory and the fp32
        output (and gradients) go back. The copies run on their own streams and are double-buffered
        against the compute, so a step's inputs stream in while the previous step computes and the
        one before it streams out (the job's throughput is set by the slower copy direction); the
        time is from the first input copy to the last output copy."""
        torch = self.torch
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        pin = {k: torch.from_numpy(self.x[k]).to(self.tdt).pin_memory() for k in self.x}
        nb = 2
        dT = [{k: torch.empty_like(self.T[k]) for k in self.T} for _ in range(nb)]
        outs = [[torch.empty_like(o) for o in [self.out] + (self.grads or [])] for _ in range(nb)]
        outs_h = [[torch.empty(o.shape, dtype=torch.float32).pin_memory() for o in outs[0]] for _ in range(nb)]
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_comp = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        start.record(s_in)
        for k in range(steps):
            b = k % nb
            with torch.cuda.stream(s_in):
                if k >= nb:
                    s_in.wait_event(ev_comp[b])  # step k - 2 has finished reading these buffers
                for name in dT[b]:
                    dT[b][name].copy_(pin[name], non_blocking=True)
                ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            if k >= nb:
                comp.wait_event(ev_out[b])  # step k - 2's outputs have left
            flush.zero_()
            self.step(T=dT[b], outs=outs[b])
            ev_comp[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                for o, oh in zip(outs[b], outs_h[b]):
                    oh.copy_(o, non_blocking=True)
                ev_out[b].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        ms = start.elapsed_time(end) / steps
        h2d = sum(pin[k].numel() * pin[k].element_size() for k in pin)
        d2h = sum(oh.numel() * 4 for oh in outs_h[0])
        return ms, h2d, d2h

    def launches_per_step(self):
        return len(self.stages)

    def release(self):
        for k in list(self.__dict__):
            if k not in ("w", "stages", "api", "torch", "dev"):
                setattr(self, k, None)
        self.torch.cuda.empty_cache()


def workload_summary(r, step_ms_list, stage_ms, peaks, peak_src, clk, n_sm, world):
    w = r.w
    ms_per_step, value = job_rate(w.tokens, world, sum(step_ms_list), len(step_ms_list))
    rec = {"workload": w.name, "metric": metric_name(w), "ms_per_step": ms_per_step, "tokens_per_s": value,
           "stage_ms": {k: round(v, 5) for k, v in stage_ms.items()}}
    if w.dtype == "bf16":
        dom = max(stage_ms, key=stage_ms.get)
        rec["roofline"] = stage_roofline(dom.split("#")[0], w, stage_ms[dom], peaks, peak_src, n_sm, clk)
        rec["path_roofline"] = path_roofline(w, ms_per_step, peaks, clk, n_sm)
    return rec


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from linear_attention_positive_b200 import api

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    peaks, peak_src = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    clocks = ClockSampler(dev.index if dev.index is not None else local)
    clocks.start()
    r = Runner(w, dev, api, torch, args.exp_poly_pct)
    step_ms, stage_ms, status = r.time(args.steps, args.warmup, flush, world, dist)
    job_ms = max_over_ranks([sum(step_ms)], world, dev)[0]
    ms_per_step, value = job_rate(w.tokens, world, job_ms, args.steps)
    e2e_ms, h2d, d2h = r.e2e(args.steps, flush, world, dist)
    e2e_ms = max_over_ranks([e2e_ms], world, dev)[0]
    headline_stage_ms = stage_ms
    x_head, W_head = (r.x, None)
    launches = r.launches_per_step() * args.steps
    r.release()

    # The other workloads of the method, each from its own event-timed loop (same steps / warm-up).
    others = {}
    if not args.headline_only:
        for k in args.also:
            if k == args.workload:
                continue
            wk = WORKLOADS[k]
            rk = Runner(wk, dev, api, torch, args.exp_poly_pct)
            sm, stg, st_k = rk.time(args.steps, args.warmup, flush, world, dist)
            sm_job = max_over_ranks([sum(sm)], world, dev)[0]
            rec = workload_summary(rk, [sm_job / args.steps] * args.steps, stg, peaks, peak_src, None, n_sm, world)
            rec["device_status"] = api.status_string(st_k)
            others[str(k)] = rec
            rk.release()
    clk = clocks.stop()
    for k, rec in others.items():  # MUFU fractions at the clock sampled over all timed loops
        if "path_roofline" in rec:
            wk = WORKLOADS[int(k)]
            rec["path_roofline"] = path_roofline(wk, rec["ms_per_step"], peaks, clk, n_sm)
            dom = max(rec["stage_ms"], key=rec["stage_ms"].get)
            rec["roofline"] = stage_roofline(dom.split("#")[0], wk, rec["stage_ms"][dom], peaks, peak_src, n_sm, clk)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    line = {
        "metric": metric_name(w), "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world),
        "e2e": {"value": job_rate(w.tokens, world, e2e_ms, 1)[1], "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "stage_ms_note": "per-kernel times come from separate steps with an event pair around every launch",
        "device_status": api.status_string(status),
    }
    if w.dtype == "bf16":
        line["stage_ms"] = {k: round(v, 5) for k, v in headline_stage_ms.items()}
        dom = max(headline_stage_ms, key=headline_stage_ms.get)
        line["roofline"] = stage_roofline(dom.split("#")[0], w, headline_stage_ms[dom], peaks, peak_src, n_sm, clk)
        line["path_roofline"] = path_roofline(w, ms_per_step, peaks, clk, n_sm)
    if clk is not None:
        line["clocks"] = clk
    if others:
        line["workloads"] = others
    if world == 1 and not args.no_cpu_baseline:
        try:
            W64 = oracle_W(w)
            n_heads = pick_sample(w, x_head, W64, budget_s=15.0)
            t0 = time.perf_counter()
            toks = oracle_sample(w, x_head, W64, [(i // w.H, i % w.H) for i in range(n_heads)])
            sec = time.perf_counter() - t0
            line["cpu_baseline"] = {"value": toks / sec, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                                    "sample": f"{n_heads} of {w.B * w.H} heads (L={w.L}), fp64 numpy oracle"}
        except Exception as exc:  # the baseline is reported, never required
            line["cpu_baseline"] = {"value": None, "error": str(exc)[:200]}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--exp-poly-pct", type=int, default=0,
                    help="percent of feature exponentials on the FMA-pipe polynomial (0: each kernel's "
                         "library default; negative: all on MUFU)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle sample after the timed region (for profiler runs)")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only --workload (not the other workloads reported under 'workloads')")
    ap.add_argument("--also", default="3,4,5,6,7,8",
                    help="comma-separated workloads timed after the headline and reported under 'workloads'")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    args.also = [int(v) for v in args.also.split(",") if v.strip()]
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
