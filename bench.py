"""Benchmark of the MoE quantization path on B200.

One step = one pass of the whole path, every op at its full-size workload:
  blockwise   fp8 1x128 on activations (16384, 4096) and 128x128 on the
              weight (14336, 4096)                        (Llama-3-8B MLP shapes)
  jagged      rowwise on grad_out^T and colwise on input, both (65536, 4096),
              G=16 Dirichlet(0.5) groups along M          (grouped-GEMM backward)
  MX 3-D      expert weights (E, 8192, 5120), E=64 by default, floor mode
  MX act      tokens (65536, 7168) rowwise 1x32, then per-group (G=64,
              Dirichlet(0.3)) 128x4 blocked layout of its E8M0 scales
Inputs are seeded synthetic tensors resident in HBM; every step moves more
than 12 GB, far above the 126 MB L2, so no flush is needed between steps.

Metric: achieved HBM GB/s = algorithmic bytes (2 B read + 1 B written per
element, plus scales) / device time, CUDA events on the launch stream, max
over ranks. Also printed: per-op us/call and GB/s, a per-shape sweep (L2
flushed before every rep), the dominant kernel's roofline against the
measured copy bandwidth, the CPU oracle on a bounded sample, an end-to-end
figure through the public API from pinned host buffers, and SM clocks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxq|reference]
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "achieved HBM GB/s and % of B200 peak per quant kernel; µs/call per shape"
WORKLOAD = "moe_quant_path"
KERNEL_NAMES = {
    "blockwise_1x128": "k_fp8_1x128",
    "blockwise_128x128": "k_fp8_128x128",
    "jagged_rowwise": "k_jagged_amax+k_jagged_cast",
    "jagged_colwise": "k_jagged_amax+k_jagged_cast",
    "mx_3d_colwise": "k_mx_3d_colwise",
    "mx_rowwise": "k_mx_1x32",
    "blocked_grouped": "k_blocked_grouped_tma",
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="mxq", choices=["mxq", "reference"])
    p.add_argument("--experts", type=int, default=64, help="E of the MX 3-D expert-weight op")
    p.add_argument("--mx3d-mode", default="floor", choices=["floor", "rceil"])
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--no-per-shape", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--reps", type=int, default=50, help="reps per shape in the per-shape sweep (cold and hot each)")
    p.add_argument("--profile-op", default=None, choices=list(Workload.OPS) + list(Workload.EXTRA),
                   help="run only this op (for single-kernel profiler captures)")
    p.add_argument("--iters", type=int, default=3, help="calls of --profile-op after one warm-up")
    return p.parse_args()


# ----------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


KERNEL_FILES = {  # source files that define each kernel (plus common.cuh)
    "k_fp8_1x128": "rowblock.cuh", "k_fp8_128x128": "rowblock.cuh", "k_mx_1x32": "rowblock.cuh",
    "k_jagged_amax": "jagged.cuh", "k_jagged_cast": "jagged.cuh", "k_mx_3d_colwise": "mx3d.cuh",
    "k_blocked_grouped": "blocked.cuh", "k_blocked_grouped_k": "blocked.cuh", "k_mx_1x32_blocked": "blocked.cuh",
    "k_fp8_blockwise_t": "blockt.cuh", "k_fp8_grouped_gemm": "gemm.cuh", "k_fp8_grouped_gemm_wgrad": "gemm.cuh",
    "k_mx_grouped_gemm": "gemm_mx.cuh", "k_jagged_single": "jagged1.cuh", "k_mx_jagged_colwise_padded": "mxj.cuh",
    "k_mx_grouped_gemm_wgrad": "mxj.cuh", "k_blocked_grouped_tma": "blockedt.cuh",
    "k_blocked_grouped_k_tma": "blockedt.cuh", "k_fp8_grouped_gemm_wgrad_2sm": "gemm2.cuh",
}


def kernel_source_hash(kernel):
    """Hash of the sources a kernel is built from: its own header and the
    shared device helpers."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp8_quantization_moe_device_b200", "csrc")
    for f in ("common.cuh", KERNEL_FILES[kernel]):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def load_traffic_capture(kernel):
    """The capture behind load_traffic(kernel), unscaled: its workload, its
    measured DRAM bytes and that workload's algorithmic bytes (None when the
    capture predates the kernel's current sources)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        parts = []
        for k in kernel.split("+"):
            e = d["kernels"][k]
            if e.get("source_hash") != kernel_source_hash(k):
                return None
            parts.append(e)
        dram = sum(e["capture_dram_bytes"] for e in parts)
        alg = sum(e["capture_algorithmic_bytes"] for e in parts[-1:])
        return {"workload": parts[-1]["capture_workload"], "dram_bytes": dram, "algorithmic_bytes": alg,
                "dram_over_algorithmic": round(dram / alg, 4), "scaled_by": parts[-1]["scaled_by"],
                "summary": parts[-1]["captured_on"]}
    except Exception:
        return None


def load_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        total = 0
        for k in kernel.split("+"):  # an op of several kernels: their sum
            e = d["kernels"][k]
            if e.get("source_hash") != kernel_source_hash(k):
                return None
            total += e["dram_bytes_per_launch"]
        return total
    except Exception:
        return None


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every ~5 ms through NVML
    during the timed region (nvidia-smi's period is too coarse for it)."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, uuid):
        self.uuid = uuid
        self.rows = []
        self.stop_flag = threading.Event()
        self.t = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv, h = self.nv, self.h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self.stop_flag.is_set():
            try:
                self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), nv.nvmlDeviceGetPowerUsage(h) / 1e3,
                                  int(get_reasons(h))))
            except Exception:
                pass
            time.sleep(0.005)

    def stop(self):
        if self.t is None:
            return None
        self.stop_flag.set()
        self.t.join(timeout=2)
        if not self.rows:
            return None
        reasons = [name for name, bit in self.REASONS if any(r[2] & bit for r in self.rows)]
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.smax,
                "sm_mhz_min": min(r[0] for r in self.rows), "reasons": reasons, "samples": len(self.rows),
                "power_w_median": round(statistics.median(r[1] for r in self.rows), 1)}


# ----------------------------------------------------------------- workload

class Workload:
    """Device tensors, outputs and the per-op launch closures of one step.
    `only` restricts construction to the tensors of one op (profiling)."""

    OPS = ("blockwise_1x128", "blockwise_128x128", "jagged_rowwise", "jagged_colwise", "mx_3d_colwise",
           "mx_rowwise", "blocked_grouped")
    # ops outside the step (the widened rows), built only when asked for by name
    EXTRA = ("blockwise_128x1_t", "blockwise_128x128_t", "blocked_grouped_k", "mx_rowwise_blocked", "grouped_gemm",
             "grouped_gemm_wgrad", "mx_grouped_gemm", "mx_jagged_colwise_padded", "mx_grouped_gemm_wgrad",
             "jagged_colwise_single_read")

    def __init__(self, dev, experts, mx3d_mode, only=None):
        import torch
        from mxfp8_quantization_moe_device_b200 import binding as mxq
        from mxfp8_quantization_moe_device_b200 import synth
        self.torch, self.mxq = torch, mxq
        self.dev = dev
        self.experts = experts
        self.mx3d_mode = mx3d_mode
        t = torch
        want = set(self.OPS if only is None else [only])
        u8 = dict(dtype=t.uint8, device=dev)
        f32 = dict(dtype=t.float32, device=dev)
        self.o = {}
        self.ops = []
        if "blockwise_1x128" in want:
            self.act = synth.blockwise_act(device=dev)
            self.o.update(act_q=t.empty(self.act.shape, **u8), act_s=t.empty((16384, 32), **f32))
            self.ops.append(("blockwise_1x128", lambda: mxq.fp8_quant_blockwise(
                self.act, 1, 128, out=self.o["act_q"], inv_scales=self.o["act_s"]), 16384 * 4096 * 3 + 16384 * 32 * 4))
        if "blockwise_128x128" in want:
            self.wt = synth.blockwise_weight(device=dev)
            self.o.update(wt_q=t.empty(self.wt.shape, **u8), wt_s=t.empty((112, 32), **f32))
            self.ops.append(("blockwise_128x128", lambda: mxq.fp8_quant_blockwise(
                self.wt, 128, 128, out=self.o["wt_q"], inv_scales=self.o["wt_s"]), 14336 * 4096 * 3 + 112 * 32 * 4))
        if want & {"jagged_rowwise", "jagged_colwise"}:
            self.grad_out, self.inp, offs16 = synth.jagged_bwd(device=dev)
            self.offs16 = offs16.to(dev)
            M, D = self.inp.shape
            jb = M * D * 3 + 16 * D * 4
            if "jagged_rowwise" in want:
                self.o.update(go_q=t.empty((D, M), **u8), go_s=t.empty((16, D), **f32))
                self.ws_r = t.empty(max(mxq.jagged_workspace_bytes(D, M, 1, D, 16, False), 1), **u8)
                self.ops.append(("jagged_rowwise", lambda: mxq.fp8_quant_jagged_rowwise(
                    self.grad_out.t(), self.offs16, out=self.o["go_q"], inv_scales=self.o["go_s"],
                    workspace=self.ws_r), jb))
            if "jagged_colwise" in want:
                self.o.update(in_q=t.empty((D, M), **u8), in_s=t.empty((16, D), **f32))
                self.ws_c = t.empty(max(mxq.jagged_workspace_bytes(M, D, D, 1, 16, True), 1), **u8)
                self.ops.append(("jagged_colwise", lambda: mxq.fp8_quant_jagged_colwise(
                    self.inp, self.offs16, out=self.o["in_q"], inv_scales=self.o["in_s"], workspace=self.ws_c), jb))
        if "mx_3d_colwise" in want:
            self.w3 = synth.mx3d_weight(experts, device=dev)
            E, N, K = self.w3.shape
            self.o.update(w3_q=t.empty((E, K, N), **u8), w3_s=t.empty((E, K, N // 32), **u8))
            self.ops.append(("mx_3d_colwise", lambda: mxq.mx_quant_3d_colwise(
                self.w3, self.mx3d_mode, out=self.o["w3_q"], scales=self.o["w3_s"]), E * N * K * 3 + E * K * N // 32))
        if want & {"mx_rowwise", "blocked_grouped"}:
            self.tok, offs64 = synth.mx_act(device=dev)
            self.offs64 = offs64.to(dev)
            T, KT = self.tok.shape
            self.o.update(tok_q=t.empty((T, KT), **u8), tok_s=t.empty((T, KT // 32), **u8))
            if "mx_rowwise" in want:
                self.ops.append(("mx_rowwise", lambda: mxq.mx_quant_rowwise(
                    self.tok, "floor", out=self.o["tok_q"], scales=self.o["tok_s"]), T * KT * 3 + T * KT // 32))
            if "blocked_grouped" in want:
                if "mx_rowwise" not in want:
                    mxq.mx_quant_rowwise(self.tok, "floor", out=self.o["tok_q"], scales=self.o["tok_s"])
                self.cap = mxq.blocked_grouped_rows_bound(T, 64)
                c4 = (KT // 32 + 3) // 4 * 4
                self.o.update(blk=t.empty(self.cap * c4, **u8), blk_starts=t.empty(64, dtype=t.int32, device=dev))
                self.ops.append(("blocked_grouped", lambda: mxq.mx_scales_to_blocked_grouped(
                    self.o["tok_s"], self.offs64, capacity_rows=self.cap, out=self.o["blk"],
                    group_row_starts=self.o["blk_starts"]), T * (KT // 32) + self.cap * c4))

        if "blockwise_128x1_t" in want:
            self.act = synth.blockwise_act(device=dev)
            self.o.update(act_qt=t.empty((4096, 16384), **u8), act_st=t.empty((4096, 128), **f32))
            self.ops.append(("blockwise_128x1_t", lambda: mxq.fp8_quant_blockwise_transposed(
                self.act, 1, out=self.o["act_qt"], inv_scales=self.o["act_st"]), 16384 * 4096 * 3 + 4096 * 128 * 4))
        if "blockwise_128x128_t" in want:
            self.wt = synth.blockwise_weight(device=dev)
            self.o.update(wt_qt=t.empty((4096, 14336), **u8), wt_st=t.empty((32, 112), **f32))
            self.ops.append(("blockwise_128x128_t", lambda: mxq.fp8_quant_blockwise_transposed(
                self.wt, 128, out=self.o["wt_qt"], inv_scales=self.o["wt_st"]), 14336 * 4096 * 3 + 32 * 112 * 4))
        if "blocked_grouped_k" in want:
            R, C = 8192, 32768
            self.sk, ok = synth.scale_sweep_k(R, C, device=dev)
            self.offs_k = ok.to(dev)
            self.o.update(blk_k=t.empty(R * (C + 32), **u8), blk_k_starts=t.empty(8, dtype=t.int32, device=dev))
            self.ops.append(("blocked_grouped_k", lambda: mxq.mx_scales_to_blocked_grouped_k(
                self.sk, self.offs_k, capacity_cols=C + 32, out=self.o["blk_k"],
                group_col_starts=self.o["blk_k_starts"]), R * C + R * (C + 32)))
        if "mx_rowwise_blocked" in want:
            self.tok, offs64 = synth.mx_act(device=dev)
            self.offs64 = offs64.to(dev)
            T, KT = self.tok.shape
            self.cap = mxq.blocked_grouped_rows_bound(T, 64)
            sbytes = self.cap * (KT // 128) * 4
            self.o.update(tok_q=t.empty((T, KT), **u8), tok_sb=t.empty(sbytes, **u8),
                          tok_sb_starts=t.empty(64, dtype=t.int32, device=dev))
            self.ops.append(("mx_rowwise_blocked", lambda: mxq.mx_quant_rowwise_blocked_grouped(
                self.tok, self.offs64, "floor", capacity_rows=self.cap, out=self.o["tok_q"], scales=self.o["tok_sb"],
                group_row_starts=self.o["tok_sb_starts"]), T * KT * 3 + sbytes))

        if "grouped_gemm" in want:
            # tokens (16384, 7168) in 16 Dirichlet(0.3) groups x 16 experts (2048, 7168): a 1 GB capture
            T, K, E, N = 16384, 7168, 16, 2048
            x = synth.normal_bf16((T, K), 1.0, seed=7, device=dev)
            w = synth.normal_bf16((E * N, K), 0.02, seed=12, device=dev)
            kk = t.tensor([K], dtype=t.int32, device=dev)
            aq, ia = mxq.fp8_quant_jagged_rowwise(x, kk)
            wq, iw = mxq.fp8_quant_jagged_rowwise(w, kk)
            del x, w
            self.g_a, self.g_ia = aq.view(t.uint8), ia.reshape(T).contiguous()
            self.g_w, self.g_iw = wq.view(t.uint8).reshape(E, N, K), iw.reshape(E, N).contiguous()
            self.g_offs = synth.dirichlet_offsets(T, E, 0.3, 8).to(dev)
            self.o.update(g_out=t.empty((T, N), dtype=t.bfloat16, device=dev))
            self.ops.append(("grouped_gemm", lambda: mxq.fp8_grouped_gemm_rowwise(
                self.g_a, self.g_ia, self.g_w, self.g_iw, self.g_offs, out=self.o["g_out"]), 2 * T * N * K))

        if "mx_grouped_gemm" in want:
            # the same MoE shape in MXFP8: codes and blocked scales from the fused MX rowwise op
            T, K, E, N = 16384, 7168, 16, 2048
            self.x_offs = synth.dirichlet_offsets(T, E, 0.3, 8).to(dev)
            x = synth.normal_bf16((T, K), 1.0, seed=7, device=dev)
            w = synth.normal_bf16((E * N, K), 0.02, seed=12, device=dev)
            qa, sa, _ = mxq.mx_quant_rowwise_blocked_grouped(x, self.x_offs, "floor")
            qw, sw, _ = mxq.mx_quant_rowwise_blocked_grouped(w, t.tensor([E * N], dtype=t.int32, device=dev), "floor")
            del x, w
            self.x_a, self.x_sa, self.x_w, self.x_sw = qa.view(t.uint8), sa, qw.view(t.uint8).reshape(E, N, K), sw
            self.o.update(x_out=t.empty((T, N), dtype=t.bfloat16, device=dev))
            self.ops.append(("mx_grouped_gemm", lambda: mxq.mx_grouped_gemm(
                self.x_a, self.x_sa, self.x_w, self.x_sw, self.x_offs, out=self.o["x_out"]), 2 * T * N * K))

        if want & {"mx_jagged_colwise_padded", "mx_grouped_gemm_wgrad", "jagged_colwise_single_read"}:
            # the jagged backward config: grad_out^T (4096, 65536) and input (65536, 4096), G=16
            go, x, offs16 = synth.jagged_bwd(device=dev)
            self.offs16 = offs16.to(dev)
            M, D = x.shape
            cap = mxq.blocked_grouped_rows_bound(M, 16)
            if "jagged_colwise_single_read" in want:
                self.inp = x
                self.o.update(in_q=t.empty((D, M), **u8), in_s=t.empty((16, D), **f32))

                def single():
                    mxq.testing_set(mxq.TESTING_FORCE_PATH, 3)
                    try:
                        mxq.fp8_quant_jagged_colwise(self.inp, self.offs16, out=self.o["in_q"],
                                                     inv_scales=self.o["in_s"])
                    finally:
                        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
                self.ops.append(("jagged_colwise_single_read", single, M * D * 3 + 16 * D * 4))
            if want & {"mx_jagged_colwise_padded", "mx_grouped_gemm_wgrad"}:
                self.inp = x
                self.o.update(mq=t.empty((D, cap), **u8), ms=t.empty(D * cap // 32, **u8))
                if "mx_jagged_colwise_padded" in want:
                    self.ops.append(("mx_jagged_colwise_padded", lambda: mxq.mx_quant_jagged_colwise_padded(
                        self.inp, self.offs16, "floor", capacity=cap, out=self.o["mq"], scales=self.o["ms"]),
                        M * D * 2 + D * cap + D * cap // 32))
                else:
                    qa, sa = mxq.mx_quant_jagged_rowwise_padded(go.t(), self.offs16, "floor", capacity=cap)
                    mxq.mx_quant_jagged_colwise_padded(x, self.offs16, "floor", capacity=cap, out=self.o["mq"],
                                                       scales=self.o["ms"])
                    self.mw = (qa.view(t.uint8), sa, self.o["mq"], self.o["ms"], M)
                    self.o.update(mw_out=t.empty((16, D, D), dtype=t.bfloat16, device=dev))
                    self.ops.append(("mx_grouped_gemm_wgrad", lambda: mxq.mx_grouped_gemm_wgrad(
                        *self.mw[:4], self.offs16, self.mw[4], out=self.o["mw_out"]), 2 * M * D * D))
            del go

        if "grouped_gemm_wgrad" in want:
            # the jagged backward config: grad_out^T (4096, 65536) and input (65536, 4096), G=16
            go, x, offs16 = synth.jagged_bwd(device=dev)
            self.offs16 = offs16.to(dev)
            M, D = x.shape
            a, ia = mxq.fp8_quant_jagged_rowwise(go.t(), self.offs16)
            b, ib = mxq.fp8_quant_jagged_colwise(x, self.offs16)
            del go, x
            self.w_a, self.w_ia, self.w_b, self.w_ib = a.view(t.uint8), ia, b.t().view(t.uint8), ib
            self.o.update(w_out=t.empty((16, D, D), dtype=t.bfloat16, device=dev))
            self.ops.append(("grouped_gemm_wgrad", lambda: mxq.fp8_grouped_gemm_wgrad(
                self.w_a, self.w_ia, self.w_b, self.w_ib, self.offs16, out=self.o["w_out"]), 2 * M * D * D))

    def step_bytes(self):
        return sum(b for _, _, b in self.ops)


def profile_op(args):
    """Run one op of the workload `iters` times after one warm-up call (for
    ncu captures of a single kernel) and print its event-timed durations."""
    import torch
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = Workload(dev, args.experts, args.mx3d_mode, only=args.profile_op)
    name, fn, nbytes = wl.ops[0]
    fn()
    torch.cuda.synchronize()
    res = []
    for _ in range(args.iters):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        us = a.elapsed_time(b) * 1e3
        res.append({"us": round(us, 2), "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1)})
    status = wl.mxq.device_status()
    print(json.dumps({"op": name, "experts": args.experts, "mode": args.mx3d_mode, "bytes": nbytes,
                      "runs": res, "status": status}))
    if status != 0:
        raise SystemExit(f"device status {status}")


def time_steps(wl, steps, warmup, per_op=True):
    """Run warmup + timed steps on the current stream; returns (total_ms,
    per-op list of per-step ms)."""
    torch = wl.torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        for _, fn, _ in wl.ops:
            fn()
    torch.cuda.synchronize()
    n = len(wl.ops)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(steps):
        ev[s][0].record(stream)
        for i, (_, fn, _) in enumerate(wl.ops):
            fn()
            ev[s][i + 1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    total = start.elapsed_time(end)
    per = [[ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)] for i in range(n)]
    return total, per


def flush_l2(torch, buf):
    buf.zero_()


def flush_l2_clean(torch, buf, sink):
    """Write `buf` (larger than L2), then read it back: L2 ends holding clean
    lines of `buf` only, so the next kernel starts cold without first having
    to write back the flush's own dirty lines."""
    buf.zero_()
    torch.sum(buf.view(torch.int64), dim=0, out=sink)


GRAPH_BELOW_BYTES = 512 << 20  # shapes timed again inside a CUDA graph


def graph_us(torch, fn, flush, calls=10, reps=5):
    """Device time per call of `fn` with the per-launch host and event
    overhead amortised away (about 5 us on B200 for a single timed call):
    two CUDA graphs, one of `calls` x (clean L2 flush, fn) and one of `calls`
    x (clean L2 flush) alone, each replayed `reps` times; the median
    difference divided by `calls`. The L2 is cold and clean before every
    call, as for "us_clean". None if the call cannot be captured."""
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                fn()
                flush()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graphs = []
        for with_fn in (True, False):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(calls):
                    flush()
                    if with_fn:
                        fn()
            g.replay()
            graphs.append(g)
        torch.cuda.synchronize()
        diffs = []
        for _ in range(reps):
            t = []
            for g in graphs:
                torch.cuda._sleep(200000)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                b.synchronize()
                t.append(a.elapsed_time(b) * 1e3)
            diffs.append((t[0] - t[1]) / calls)
        del graphs
        return round(statistics.median(diffs), 3)
    except Exception:
        torch.cuda.synchronize()
        return None


def per_shape_sweep(wl, reps):
    """us/call and GB/s per config shape after 5 warm-up calls: the median of
    `reps` calls with the L2 flushed (256 MB write) before each ("us"); the
    median of `reps` calls after the same write followed by a read of the
    flush buffer, so that the L2 is cold but holds no dirty lines the call
    would first have to write back ("us_clean"); the median of `reps`
    back-to-back calls with a hot L2 ("us_hot", labelled as such); the
    median host time to enqueue one call ("enqueue_us"); and, for shapes
    under 512 MB, the per-call device time from CUDA graphs with a clean L2
    flush before every call ("us_graph", see graph_us), which a single timed
    call overstates by the launch and event overhead (about 5 us on B200)."""
    torch, mxq = wl.torch, wl.mxq
    from mxfp8_quantization_moe_device_b200 import synth
    dev = wl.dev
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)
    peak, _ = load_peaks()
    rows = []

    def run(name, shape, fn, nbytes):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ts, clean, hot, enq = [], [], [], []
        for mode in ("cold", "clean", "hot"):
            for _ in range(reps):
                if mode == "cold":
                    flush_l2(torch, flush)
                elif mode == "clean":
                    flush_l2_clean(torch, flush, sink)
                else:
                    # keep the GPU busy (~100 us, no memory traffic) while the
                    # host enqueues, so that the events time the call alone
                    torch.cuda._sleep(200000)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                h0 = time.perf_counter()
                fn()
                h1 = time.perf_counter()
                b.record()
                b.synchronize()
                {"cold": ts, "clean": clean, "hot": hot}[mode].append(a.elapsed_time(b) * 1e3)
                enq.append((h1 - h0) * 1e6)
        us = statistics.median(ts)
        gbs = nbytes / (us * 1e-6) / 1e9
        usc = statistics.median(clean)
        row = {"op": name, "shape": shape, "us": round(us, 3), "GB/s": round(gbs, 1),
               "frac_measured": round(gbs / peak, 4), "frac_8TBs": round(gbs / 8000.0, 4),
               "us_clean": round(usc, 3), "frac_measured_clean": round(nbytes / (usc * 1e-6) / 1e9 / peak, 4),
               "us_hot": round(statistics.median(hot), 3), "enqueue_us": round(statistics.median(enq), 1)}
        if nbytes < GRAPH_BELOW_BYTES:
            row["us_graph"] = graph_us(torch, fn, lambda: flush_l2_clean(torch, flush, sink))
            if row["us_graph"]:
                row["frac_measured_graph"] = round(nbytes / (row["us_graph"] * 1e-6) / 1e9 / peak, 4)
        rows.append(row)

    run.rows = rows

    # tiny jagged
    a, offs = synth.tiny_jagged(device=dev)
    offs = offs.to(dev)
    run("jagged_colwise", "(256,512) G=4", lambda: mxq.fp8_quant_jagged_colwise(a, offs), 256 * 512 * 3 + 4 * 512 * 4)
    run("jagged_rowwise", "(512,256)^T G=4", lambda: mxq.fp8_quant_jagged_rowwise(a.t(), offs), 256 * 512 * 3 + 4 * 512 * 4)
    by = {n: (f, b) for n, f, b in wl.ops}
    run("blockwise_1x128", "(16384,4096)", *by["blockwise_1x128"])
    run("blockwise_128x128", "(14336,4096)", *by["blockwise_128x128"])
    run("jagged_rowwise", "(4096,65536)^T G=16", *by["jagged_rowwise"])
    run("jagged_colwise", "(65536,4096) G=16", *by["jagged_colwise"])
    E = wl.w3.shape[0]
    for e in [x for x in (1, 2, 4, 8, 16, 64) if x <= E]:
        w = wl.w3[:e]
        for mode in ("floor", "rceil"):
            out = wl.o["w3_q"][:e]
            sc = wl.o["w3_s"][:e]
            run("mx_3d_colwise", f"({e},8192,5120) {mode}",
                lambda w=w, mode=mode, out=out, sc=sc: mxq.mx_quant_3d_colwise(w, mode, out=out, scales=sc),
                e * 8192 * 5120 * 3 + e * 5120 * 256)
    for mode in ("floor", "rceil"):
        run("mx_rowwise", f"(65536,7168) {mode}",
            lambda mode=mode: mxq.mx_quant_rowwise(wl.tok, mode, out=wl.o["tok_q"], scales=wl.o["tok_s"]),
            65536 * 7168 * 3 + 65536 * 224)
    run("blocked_grouped", "(65536,224) G=64", *by["blocked_grouped"])
    for R in (8192, 5120, 7168, 2048):
        for C in (512, 1024, 2048, 4096, 32768):
            s, o = synth.scale_sweep(R, C, device="cpu")
            s, o = s.to(dev), o.to(dev)
            cap = mxq.blocked_grouped_rows_bound(R, 8)
            out = torch.empty(cap * C, dtype=torch.uint8, device=dev)
            st = torch.empty(8, dtype=torch.int32, device=dev)
            run("blocked_grouped", f"({R},{C}) G=8",
                lambda s=s, o=o, cap=cap, out=out, st=st: mxq.mx_scales_to_blocked_grouped(
                    s, o, capacity_rows=cap, out=out, group_row_starts=st),
                R * C + cap * C)
    # blockwise with transposed output: activations 128x1, weight 128x128
    qt_a = torch.empty(4096 * 16384, dtype=torch.uint8, device=dev)
    it_a = torch.empty((4096, 128), dtype=torch.float32, device=dev)
    run("blockwise_128x1_t", "(16384,4096)",
        lambda: mxq.fp8_quant_blockwise_transposed(wl.act, 1, out=qt_a.view(4096, 16384), inv_scales=it_a),
        16384 * 4096 * 3 + 4096 * 128 * 4)
    qt_w = torch.empty(4096 * 14336, dtype=torch.uint8, device=dev)
    it_w = torch.empty((32, 112), dtype=torch.float32, device=dev)
    run("blockwise_128x128_t", "(14336,4096)",
        lambda: mxq.fp8_quant_blockwise_transposed(wl.wt, 128, out=qt_w.view(4096, 14336), inv_scales=it_w),
        14336 * 4096 * 3 + 32 * 112 * 4)
    del qt_a, qt_w
    # groups along K: the pages' sweep shapes, G=8 along the columns, capacity C + 4G
    for R in (8192, 5120, 7168, 2048):
        for C in (512, 1024, 2048, 4096, 32768):
            s, o = synth.scale_sweep_k(R, C, device="cpu")
            s, o = s.to(dev), o.to(dev)
            out = torch.empty(R * (C + 32), dtype=torch.uint8, device=dev)
            st = torch.empty(8, dtype=torch.int32, device=dev)
            run("blocked_grouped_k", f"({R},{C}) G=8",
                lambda s=s, o=o, out=out, st=st: mxq.mx_scales_to_blocked_grouped_k(
                    s, o, capacity_cols=C + 32, out=out, group_col_starts=st),
                R * C + R * (C + 32))
    # MX rowwise quantization writing blocked scales directly (a5 + a6 fused)
    tc = 7168 // 128
    for mode in ("floor", "rceil"):
        sbuf = torch.empty(wl.cap * tc * 4, dtype=torch.uint8, device=dev)
        st = torch.empty(64, dtype=torch.int32, device=dev)
        run("mx_rowwise_blocked", f"(65536,7168) G=64 {mode}",
            lambda mode=mode, sbuf=sbuf, st=st: mxq.mx_quant_rowwise_blocked_grouped(
                wl.tok, wl.offs64, mode, capacity_rows=wl.cap, out=wl.o["tok_q"], scales=sbuf,
                group_row_starts=st),
            65536 * 7168 * 3 + wl.cap * tc * 4)
    # grouped GEMM on the tensor cores, fed by the rowwise quantization:
    # tokens (65536, 7168) in the 64 Dirichlet(0.3) groups x 64 experts (2048, 7168)
    # the tensor-core rows run last and draw the most power: their clocks
    # are sampled on their own and attached to each of them
    clk = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    clk.start()
    g_rows = gemm_rows(wl, flush, reps)
    g_rows += mx_wgrad_rows(wl, run, flush, reps)
    g_rows += grouped_mm_rows(wl, flush, max(reps // 5, 5))
    g_clocks = clk.stop()
    sus, sus_kind = _fp8_peak_sustained()
    for r in g_rows:
        if "TFLOP/s" in r:
            r["clocks_tensor_rows"] = g_clocks
            if "frac_fp8_peak" in r:  # long loops under the power cap: the sustained peak applies too
                r["frac_fp8_peak_sustained"] = round(r["TFLOP/s"] / sus, 4)
                r["peak_sustained_TFLOP/s"] = round(sus, 1)
                r["peak_sustained_kind"] = sus_kind
    rows += g_rows
    rows += jagged_extra_rows(wl, run)
    del flush
    return rows


def jagged_extra_rows(wl, run):
    """The jagged colwise op on its single-read kernel (forced; the automatic
    choice is the two-pass kernels), labelled as such."""
    mxq = wl.mxq
    if not hasattr(wl, "inp"):
        return []
    rows = []
    M, D = wl.inp.shape
    mxq.testing_set(mxq.TESTING_FORCE_PATH, 3)
    try:
        before = len(run.rows)
        run("jagged_colwise_single_read", "(65536,4096) G=16",
            lambda: mxq.fp8_quant_jagged_colwise(wl.inp, wl.offs16), M * D * 3 + 16 * D * 4)
        rows = run.rows[before:]
        del run.rows[before:]
    finally:
        mxq.testing_set(mxq.TESTING_FORCE_PATH, 0)
    return rows


def mx_wgrad_rows(wl, run, flush, reps):
    """The MXFP8 weight gradient on the jagged backward config: MX
    quantization of grad_out^T and of the input along each group's tokens
    (groups padded to 128 tokens, blocked scales), then the block-scaled
    weight-gradient GEMM (16, 4096, 4096) against the FP8 dense peak."""
    torch, mxq = wl.torch, wl.mxq
    if not hasattr(wl, "inp"):
        return []
    M, D = wl.inp.shape
    G = 16
    cap = mxq.blocked_grouped_rows_bound(M, G)
    qa = torch.empty((D, cap), dtype=torch.uint8, device=wl.dev)
    sa = torch.empty(D * cap // 32, dtype=torch.uint8, device=wl.dev)
    qb = torch.empty((D, cap), dtype=torch.uint8, device=wl.dev)
    sb = torch.empty(D * cap // 32, dtype=torch.uint8, device=wl.dev)
    nbytes = M * D * 2 + D * cap + D * cap // 32
    before = len(run.rows)
    run("mx_jagged_rowwise_padded", "(4096,65536)^T G=16 floor",
        lambda: mxq.mx_quant_jagged_rowwise_padded(wl.grad_out.t(), wl.offs16, "floor", capacity=cap, out=qa,
                                                   scales=sa), nbytes)
    run("mx_jagged_colwise_padded", "(65536,4096) G=16 floor",
        lambda: mxq.mx_quant_jagged_colwise_padded(wl.inp, wl.offs16, "floor", capacity=cap, out=qb, scales=sb),
        nbytes)
    rows = run.rows[before:]
    del run.rows[before:]
    out = torch.empty((G, D, D), dtype=torch.bfloat16, device=wl.dev)
    fn = lambda: mxq.mx_grouped_gemm_wgrad(qa, sa, qb, sb, wl.offs16, M, out=out)
    us = _median_us(torch, fn, max(reps // 5, 3), flush)
    tf = 2.0 * M * D * D / (us * 1e-6) / 1e12
    peak, kind = _fp8_peak()
    rows.append({"op": "mx_grouped_gemm_wgrad", "shape": f"({D},{cap})x({D},{cap}) G=16 -> (16,{D},{D})",
                 "us": round(us, 3), "TFLOP/s": round(tf, 1), "frac_fp8_peak": round(tf / peak, 4),
                 "peak_TFLOP/s": round(peak, 1), "peak_kind": kind})
    del qa, qb, out
    return rows


def _fp8_peak_sustained():
    """FP8 dense peak for kernels timed inside a long loop under the power
    cap: the measured sustained bf16 GEMM rate times the nominal ratio 2."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 2.0 * float(json.load(f)["bf16_tflops_sustained"]), "measured sustained bf16 x 2"
    except Exception:
        return 2.0 * 1390.0, "fallback sustained bf16 x 2"


def _fp8_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 2"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 x 2"


def _median_us(torch, fn, reps, flush):
    """Median device time of `fn` over `reps` calls, L2 flushed before each."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush_l2(torch, flush)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    return statistics.median(ts)


def grouped_mm_rows(wl, flush, reps):
    """One forward + backward of the differentiable grouped matmuls at the
    shapes of the page "[scaled grouped mm] integrate triton kernels into
    differentiable scaled grouped mm" (Performance): tokens A (M, 4096) with
    M in {256, 4096, 65536} x experts B (E, 4096, 4096) with E in {4, 8, 16},
    the tokens split equally among the experts (the page does not give its
    group sizes). Device time of out = mm(a, w, offs); out.backward(dy), and
    its TFLOP/s over the three GEMMs (6 M N K)."""
    torch = wl.torch
    from mxfp8_quantization_moe_device_b200 import synth
    from mxfp8_quantization_moe_device_b200.autograd import fp8_grouped_mm, mx_grouped_mm
    dev = wl.dev
    rows = []
    K = N = 4096
    for M in (256, 4096, 65536):
        a = synth.row_scaled_normal_bf16(M, K, seed=81, device=dev).requires_grad_(True)
        dy = synth.row_scaled_normal_bf16(M, N, seed=82, device=dev)
        for E in (4, 8, 16):
            w = synth.normal_bf16((E, N, K), 0.02, 83, device=dev).requires_grad_(True)
            offs = torch.arange(M // E, M + 1, M // E, dtype=torch.int32).to(dev)
            for name, mm in (("fp8_grouped_mm", lambda: fp8_grouped_mm(a, w, offs)),
                             ("mx_grouped_mm", lambda: mx_grouped_mm(a, w, offs, "floor"))):
                def step(mm=mm):
                    a.grad, w.grad = None, None
                    mm().backward(dy)
                us = _median_us(torch, step, reps, flush)
                rows.append({"op": name + "_fwd_bwd", "shape": f"A ({M},{K}) x B ({E},{N},{K})", "us": round(us, 1),
                             "TFLOP/s": round(6.0 * M * N * K / (us * 1e-6) / 1e12, 1)})
            del w
        del a, dy
    return rows


def gemm_rows(wl, flush, reps):
    """TFLOP/s of fp8_grouped_gemm_rowwise on the MoE shape, against the FP8
    dense peak taken as the measured bf16 GEMM peak times the nominal FP8/bf16
    ratio of 2."""
    torch, mxq = wl.torch, wl.mxq
    from mxfp8_quantization_moe_device_b200 import synth
    dev = wl.dev
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        kind = "measured bf16 x 2"
    except Exception:
        bf16, kind = 1590.0, "fallback bf16 x 2"
    fp8_peak = 2.0 * bf16
    T, K = wl.tok.shape
    E, N = 64, 2048
    kk = torch.tensor([K], dtype=torch.int32, device=dev)
    aq, ia = mxq.fp8_quant_jagged_rowwise(wl.tok, kk)
    w = synth.normal_bf16((E * N, K), 0.02, seed=12, device=dev)
    wq, iw = mxq.fp8_quant_jagged_rowwise(w, kk)
    del w
    aq, ia = aq.view(torch.uint8), ia.reshape(T).contiguous()
    wq, iw = wq.view(torch.uint8).reshape(E, N, K), iw.reshape(E, N).contiguous()
    out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    fn = lambda: mxq.fp8_grouped_gemm_rowwise(aq, ia, wq, iw, wl.offs64, out=out)
    for _ in range(5):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush_l2(torch, flush)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    us = statistics.median(ts)
    flops = 2.0 * T * N * K
    tf = flops / (us * 1e-6) / 1e12
    rows = [{"op": "fp8_grouped_gemm", "shape": f"({T},{K}) G=64 x (64,{N},{K})", "us": round(us, 3),
             "TFLOP/s": round(tf, 1), "frac_fp8_peak": round(tf / fp8_peak, 4), "peak_TFLOP/s": round(fp8_peak, 1),
             "peak_kind": kind}]
    del aq, wq
    # the same shape in MXFP8: MX rowwise codes with blocked scales (one
    # fused kernel per operand) into the block-scaled grouped GEMM
    qa, sa, _ = mxq.mx_quant_rowwise_blocked_grouped(wl.tok, wl.offs64, "floor")
    w = synth.normal_bf16((E * N, K), 0.02, seed=12, device=dev)
    qw, sw, _ = mxq.mx_quant_rowwise_blocked_grouped(w, torch.tensor([E * N], dtype=torch.int32, device=dev), "floor")
    del w
    qa, qw = qa.view(torch.uint8), qw.view(torch.uint8).reshape(E, N, K)
    fn = lambda: mxq.mx_grouped_gemm(qa, sa, qw, sw, wl.offs64, out=out)
    for _ in range(5):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush_l2(torch, flush)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    us = statistics.median(ts)
    tf = flops / (us * 1e-6) / 1e12
    rows.append({"op": "mx_grouped_gemm", "shape": f"({T},{K}) G=64 x (64,{N},{K})", "us": round(us, 3),
                 "TFLOP/s": round(tf, 1), "frac_fp8_peak": round(tf / fp8_peak, 4), "peak_TFLOP/s": round(fp8_peak, 1),
                 "peak_kind": kind})
    del qa, qw, out
    # weight gradient of the jagged backward config: grad_out^T (4096, 65536)
    # rowwise and input (65536, 4096) colwise, G=16, -> (16, 4096, 4096)
    if hasattr(wl, "grad_out"):
        M, D = wl.inp.shape
        a, ia = mxq.fp8_quant_jagged_rowwise(wl.grad_out.t(), wl.offs16)
        b, ib = mxq.fp8_quant_jagged_colwise(wl.inp, wl.offs16)
        a, b = a.view(torch.uint8), b.t().view(torch.uint8)
        gw = torch.empty((16, D, D), dtype=torch.bfloat16, device=dev)
        fn = lambda: mxq.fp8_grouped_gemm_wgrad(a, ia, b, ib, wl.offs16, out=gw)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(max(reps // 5, 3)):
            flush_l2(torch, flush)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        us = statistics.median(ts)
        tf = 2.0 * M * D * D / (us * 1e-6) / 1e12
        rows.append({"op": "fp8_grouped_gemm_wgrad", "shape": f"({D},{M})x({D},{M}) G=16 -> (16,{D},{D})",
                     "us": round(us, 3), "TFLOP/s": round(tf, 1), "frac_fp8_peak": round(tf / fp8_peak, 4),
                     "peak_TFLOP/s": round(fp8_peak, 1), "peak_kind": kind})
    return rows


# ----------------------------------------------------------------- oracle side

def oracle_samples(wl):
    """Bounded host samples of every op of the step, with the algorithmic
    bytes each sample stands for: (name, fn, sample_bytes, full_bytes)."""
    import numpy as np
    import oracle
    torch = wl.torch

    def words(t):
        return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    full = {n: b for n, _, b in wl.ops}
    act = words(wl.act[:4096])
    wt = words(wl.wt[:2048])
    go = words(wl.grad_out[:, :768])       # (65536, <=768): rowwise on its transpose
    inp = words(wl.inp[:, :768])
    w3s = wl.w3[0, :, :1280]
    w3 = words(w3s).reshape(1, w3s.shape[0], w3s.shape[1])
    tok = words(wl.tok[:2048])
    from mxfp8_quantization_moe_device_b200 import synth
    scales = synth.uniform_u8((65536, 224), 0, 254, seed=9).numpy()  # synthetic, never a GPU output
    offs16 = wl.offs16.cpu().numpy()
    offs64 = wl.offs64.cpu().numpy()
    M, C = go.shape
    return [
        ("blockwise_1x128", lambda: oracle.fp8_quant_blockwise(act, 1, 128), act.size * 3 + act.size // 128 * 4,
         full["blockwise_1x128"]),
        ("blockwise_128x128", lambda: oracle.fp8_quant_blockwise(wt, 128, 128), wt.size * 3 + wt.size // 16384 * 4,
         full["blockwise_128x128"]),
        ("jagged_rowwise", lambda: oracle.fp8_quant_jagged_rowwise(go.reshape(-1), C, M, 1, C, offs16),
         go.size * 3 + 16 * C * 4, full["jagged_rowwise"]),
        ("jagged_colwise", lambda: oracle.fp8_quant_jagged_colwise(inp.reshape(-1), M, C, C, 1, offs16),
         inp.size * 3 + 16 * C * 4, full["jagged_colwise"]),
        ("mx_3d_colwise", lambda: oracle.mx_quant_3d_colwise(w3, 0 if wl.mx3d_mode == "floor" else 1),
         w3.size * 3 + w3.size // 32, full["mx_3d_colwise"]),
        ("mx_rowwise", lambda: oracle.mx_quant_rowwise(tok, 0), tok.size * 3 + tok.size // 32, full["mx_rowwise"]),
        ("blocked_grouped", lambda: oracle.mx_scales_to_blocked_grouped(scales, offs64, wl.cap),
         full["blocked_grouped"], full["blocked_grouped"]),
    ]


def host_description():
    """The host the oracle runs on: core count and CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"nproc": usable, "cpu_count": os.cpu_count(), "cpu_model": model}


def run_oracle_samples(samples):
    """Time each sample once; estimate the oracle's time for the full step
    from each op's per-byte rate. Returns (GB/s, seconds spent, per-op)."""
    est = 0.0
    spent = 0.0
    per = {}
    for name, fn, sb, fb in samples:
        t0 = time.perf_counter()
        fn()
        dt = time.perf_counter() - t0
        spent += dt
        est += dt * fb / sb
        per[name] = round(sb / dt / 1e9, 4)
    total = sum(fb for _, _, _, fb in samples)
    return total / est / 1e9, spent, per


SAMPLE_DESC = ("single-threaded C oracle on a slice of every op: act rows 0-4095, weight rows 0-2047, "
               "grad_out/input columns 0-767 (all 65536 rows, G=16), expert 0 columns 0-1279, tokens rows 0-2047, "
               "the full (65536,224) scale matrix; each op's time scaled to its full-size bytes")


REF_SAMPLE_DESC = ("single-threaded C oracle, one pass per step over a slice of every op: act rows 0-511, "
                   "weight rows 0-255, grad_out/input columns 0-95 (all 65536 rows, G=16), expert 0 columns "
                   "0-159, tokens rows 0-255, the full (65536,224) scale matrix; each op's time scaled to its "
                   "full-size bytes")


# ----------------------------------------------------------------- e2e

# inputs (host -> device) and outputs (device -> host) of each op of the step
E2E_IO = {
    "blockwise_1x128": (("act",), ("act_q", "act_s")),
    "blockwise_128x128": (("wt",), ("wt_q", "wt_s")),
    "jagged_rowwise": (("grad_out", "offs16"), ("go_q", "go_s")),
    "jagged_colwise": (("inp",), ("in_q", "in_s")),
    "mx_3d_colwise": (("w3",), ("w3_q", "w3_s")),
    "mx_rowwise": (("tok", "offs64"), ("tok_q", "tok_s")),
    "blocked_grouped": ((), ("blk", "blk_starts")),
}


def run_e2e(wl, steps):
    """The same step through the public API from pinned host buffers: every
    step copies every op's inputs host->device (the group offsets included),
    runs every op, and copies every output back to pinned host memory, all
    inside the timed region. Three streams (copy in, compute, copy out) with
    events: an op's outputs travel back while the next op's inputs come in
    (PCIe is full duplex), and a step's copies into a buffer wait for the
    previous step's use of it."""
    torch = wl.torch
    host_in = {}
    for name in ("act", "wt", "grad_out", "inp", "w3", "tok", "offs16", "offs64"):
        t = getattr(wl, name)
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        host_in[name] = h
    host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in wl.o.items()}
    bi = sum(h.numel() * h.element_size() for h in host_in.values())
    bo = sum(h.numel() * h.element_size() for h in host_out.values())
    # the largest transfer first: its results return while the rest come in
    order = sorted(wl.ops, key=lambda op: op[0] != "mx_3d_colwise")
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    done_c = {n: None for n, _, _ in order}   # last compute of each op
    done_o = {n: None for n, _, _ in order}   # last copy-out of each op
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(steps):
        for name, fn, _ in order:
            ins, outs = E2E_IO[name]
            if done_c[name] is not None:
                s_in.wait_event(done_c[name])      # the previous step has read these inputs
            with torch.cuda.stream(s_in):
                for k in ins:
                    getattr(wl, k).copy_(host_in[k], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            s_c.wait_event(ev_in)
            if done_o[name] is not None:
                s_c.wait_event(done_o[name])       # the previous step's outputs are back on the host
            with torch.cuda.stream(s_c):
                fn()
            ev_c = torch.cuda.Event()
            ev_c.record(s_c)
            done_c[name] = ev_c
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                for k in outs:
                    host_out[k].copy_(wl.o[k], non_blocking=True)
            ev_o = torch.cuda.Event()
            ev_o.record(s_out)
            done_o[name] = ev_o
    s_in.wait_stream(s_c)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # the results that reached the host are the device's (first and last MB of each)
    ok = True
    for k, h in host_out.items():
        d = wl.o[k].reshape(-1).view(torch.uint8) if wl.o[k].element_size() == 1 else wl.o[k].reshape(-1)
        hv = h.reshape(-1).view(torch.uint8) if h.element_size() == 1 else h.reshape(-1)
        n = min(d.numel(), 1 << 20)
        ok = ok and torch.equal(hv[:n], d[:n].cpu()) and torch.equal(hv[-n:], d[-n:].cpu())
    del host_in, host_out
    return ms, bi, bo, ok


# ----------------------------------------------------------------- ranks

def max_over_ranks(x, device, world):
    """Max of a per-rank float over all ranks (the timing rule: the slowest
    replica sets the step time). Every rank must call it."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(step_bytes, steps, total_ms_max, world):
    """Whole-job GB/s: every replica moves step_bytes per step."""
    return world * step_bytes * steps / (total_ms_max * 1e-3) / 1e9


# ----------------------------------------------------------------- main

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and "CUDA_VISIBLE_DEVICES" not in os.environ:
        # one GPU per process: this process sees only its own device as cuda:0
        os.environ["CUDA_VISIBLE_DEVICES"] = str(local)
    import torch

    if args.profile_op:
        return profile_op(args)
    if args.impl == "reference":
        return main_reference(args, world, rank)

    import torch.distributed as dist
    if world > 1:
        dev_index = 0 if os.environ.get("CUDA_VISIBLE_DEVICES", "").count(",") == 0 else local
        torch.cuda.set_device(dev_index)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    from mxfp8_quantization_moe_device_b200 import binding as mxq
    mxq.lib()

    wl = Workload(dev, args.experts, args.mx3d_mode)
    step_bytes = wl.step_bytes()
    peak, peak_kind = load_peaks()

    clk = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk.start()
    total_ms, per = time_steps(wl, args.steps, args.warmup)
    clocks = clk.stop()
    status = mxq.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")

    total_ms = max_over_ranks(total_ms, dev, world)
    ms_per_step = total_ms / args.steps
    value = aggregate_value(step_bytes, args.steps, total_ms, world)

    per_op = {}
    for (name, _, nbytes), ts in zip(wl.ops, per):
        us = statistics.mean(ts) * 1e3
        gbs = nbytes / (us * 1e-6) / 1e9
        per_op[name] = {"us": round(us, 2), "GB/s": round(gbs, 1), "frac_measured": round(gbs / peak, 4),
                        "frac_8TBs": round(gbs / 8000.0, 4), "bytes": nbytes, "share": 0.0}
    tot_us = sum(v["us"] for v in per_op.values())
    for v in per_op.values():
        v["share"] = round(v["us"] / tot_us, 4)
    dom = max(per_op, key=lambda k: per_op[k]["us"])
    dom_bytes = per_op[dom]["bytes"]
    achieved = per_op[dom]["GB/s"]
    roofline = {"bound": "hbm", "kernel": KERNEL_NAMES[dom], "op": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": dom_bytes, "traffic": load_traffic(KERNEL_NAMES[dom]),
                "traffic_capture": load_traffic_capture(KERNEL_NAMES[dom])}

    out = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3 (fp32 scale math)",
           "data": "synthetic (seeded; shapes and distributions of the source pages' workloads)",
           "config": {"workload": WORKLOAD,
                      "ops": ["fp8 blockwise 1x128 (16384,4096)", "fp8 blockwise 128x128 (14336,4096)",
                              "fp8 jagged rowwise grad_out^T (65536,4096) G=16",
                              "fp8 jagged colwise input (65536,4096) G=16",
                              f"mx 3d colwise ({args.experts},8192,5120) {args.mx3d_mode}",
                              "mx rowwise 1x32 (65536,7168) floor",
                              "mx scales to blocked grouped (65536,224) G=64"],
                      "step_bytes": step_bytes, "parallelism": f"replicas x{world}",
                      "l2": "no flush: inputs larger than L2 (each step moves >12 GB)"},
           "roofline": roofline, "per_op": per_op, "gpu_launches": sum(KERNEL_NAMES[n].count("+") + 1 for n, _, _ in wl.ops) * args.steps,
           "clocks": clocks}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        samples = oracle_samples(wl)
        gbs, spent, per_o = run_oracle_samples(samples)
        out["cpu_baseline"] = {"value": round(gbs, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": SAMPLE_DESC, "seconds": round(spent, 2), "per_op_GB/s": per_o,
                               "extrapolated_from_sample": True, "host": host_description()}
    if not args.no_e2e:
        ms, bi, bo, ok = run_e2e(wl, max(1, args.e2e_steps))
        ms = max_over_ranks(ms, dev, world)
        out["e2e"] = {"value": round(world * step_bytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                      "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(ms, 3),
                      "steps": max(1, args.e2e_steps), "results_match_device": ok}
    if not args.no_per_shape and rank == 0:
        clk_ps = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
        clk_ps.start()
        out["per_shape"] = per_shape_sweep(wl, args.reps)
        out["per_shape_clocks"] = clk_ps.stop()
    if world > 1:
        dist.barrier()
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()


def main_reference(args, world, rank):
    """The CPU oracle as the reference arm: rank 0 times it on bounded samples
    of the same workload, one pass over the samples per step."""
    if rank != 0:
        return
    import torch
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        torch.cuda.set_device(dev)
    wl = RefWorkload(dev, args.experts, args.mx3d_mode)
    samples = wl.samples
    for _ in range(args.warmup):
        samples[0][1]()
    times = []
    t0 = time.perf_counter()
    vals = []
    for _ in range(args.steps):
        gbs, spent, _ = run_oracle_samples(samples)
        vals.append(gbs)
        times.append(spent)
    value = statistics.median(vals)
    total = sum(fb for _, _, _, fb in samples)
    # the oracle runs a bounded slice per step; ms_per_step is the full
    # step's bytes at the rate measured on that slice (flagged as such), and
    # sample_ms_per_step is the slice's own measured time
    out = {"metric": METRIC, "impl": "reference", "value": round(value, 5), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / (value * 1e9) * 1e3, 1),
           "extrapolated_from_sample": True, "sample_ms_per_step": round(statistics.median(times) * 1e3, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3 (fp32 scale math)",
           "data": "synthetic (seeded)",
           "config": {"workload": WORKLOAD, "step_bytes": total, "parallelism": "single-threaded CPU oracle"},
           "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                            "sample": REF_SAMPLE_DESC, "extrapolated_from_sample": True,
                            "host": host_description()},
           "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "wall_s": round(time.perf_counter() - t0, 1)}
    print(json.dumps(out))


class RefWorkload:
    """Host-only view of the workload for the reference arm: the same seeded
    tensors (drawn on the GPU when there is one), sliced to the oracle samples."""

    def __init__(self, dev, experts, mx3d_mode):
        import torch
        from mxfp8_quantization_moe_device_b200 import synth
        self.torch = torch
        self.mx3d_mode = mx3d_mode
        self.dev = dev
        self.act = synth.blockwise_act(device=dev, rows=512)
        self.wt = synth.blockwise_weight(device=dev, rows=256)
        go, inp, offs16 = synth.jagged_bwd(device=dev)
        self.grad_out, self.inp = go[:, :96].contiguous(), inp[:, :96].contiguous()
        del go, inp
        self.offs16 = offs16
        self.w3 = synth.mx3d_weight(1, device=dev)[:, :, :160].contiguous()
        tok, offs64 = synth.mx_act(device=dev)
        self.tok = tok[:256].contiguous()
        self.offs64 = offs64
        self.cap = 128 * ((65536 + 127 * 64) // 128)
        E = experts
        full = {"blockwise_1x128": 16384 * 4096 * 3 + 16384 * 32 * 4,
                "blockwise_128x128": 14336 * 4096 * 3 + 112 * 32 * 4,
                "jagged_rowwise": 65536 * 4096 * 3 + 16 * 4096 * 4,
                "jagged_colwise": 65536 * 4096 * 3 + 16 * 4096 * 4,
                "mx_3d_colwise": E * 8192 * 5120 * 3 + E * 5120 * 256,
                "mx_rowwise": 65536 * 7168 * 3 + 65536 * 224,
                "blocked_grouped": 65536 * 224 + self.cap * 224}
        self.ops = [(k, None, v) for k, v in full.items()]
        self.samples = oracle_samples(self)


if __name__ == "__main__":
    main()
