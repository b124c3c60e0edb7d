"""Benchmark of the GDN-2 chunkwise recurrence on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: forward tokens/s on the single-layer workload of the pages' 1.3B
model (B=8, H=16, T=4096, d_k=d_v=128, bf16 inputs, fp32 log-decay and state;
a token covers all 16 heads).  A step is one gdn2_chunk_fwd call over the
batch, inputs resident in HBM (1.09 GB per step, larger than the 126 MB L2, so
no flush is needed).  The same line carries the forward+backward figure on the
same batch (`fwd_bwd`: a training step, gdn2_chunk_fwd_save + gdn2_chunk_bwd_saved, the
forward recording the chunk-boundary states the backward needs; `bwd_ms` is the standalone
backward, which recomputes them), the decode figure (`decode`, 256 sequences, 1024
steps) and the roofline fraction of each, plus:

* `e2e`: the same forward through the C-ABI call with host buffers (gdn2_chunk_fwd_host):
  pinned-host inputs copied in and o/S_T copied out inside the timed region, pipelined with
  the kernels by batch rows;
* `cpu_baseline`: the fp64 oracle timed on a bounded sample on the host cores;
* `clocks`: SM clock and throttle reasons sampled during the timed regions;
* `sweep`: forward throughput at 65,536 tokens per call for T = 2K ... 32K (B = 32 ... 2),
  with the number of (batch, head) chains each shape gives the 148 SMs (`scan`: the shape
  takes the chunk-parallel scan, for at most 48 chains);
* `varlen`: the headline's 32,768 tokens as 16 packed sequences of log-uniform length
  (256 ... 8192, seeded), through gdn2_chunk_fwd_varlen / gdn2_chunk_bwd_varlen;
* `scalar_decay`: the headline batch with one log decay per (token, head) through
  gdn2_chunk_fwd_gated (the tensor-core forward's scalar-decay path);
* `kda`, `gated_deltanet`: the headline batch with scalar b = w = beta (and, for Gated
  DeltaNet, a scalar decay) through the gated forward and backward, whose kernels read the
  scalar gates as they are;
* `d64`: the same model width with head size 64 (H = 32), forward and backward;
* `prologue`: raw q, k and gate logits, with the input prologue (L2-normalised q, k;
  sigmoid b, w) fused into the tensor-core forward, against the same prologue run as a
  separate pass (gdn2_prologue) before the plain forward.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
independent (batch, head) sequences; there is no collective on the data path
(weak scaling).  Timing is by CUDA events, max over ranks.

`--impl reference` times the fp64 CPU oracle (the only reference this method
has: the pages publish no code) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic_inputs import DECODE_WORKLOAD, WORKLOADS, DecodeStream, make_inputs  # noqa: E402

METRIC = "GDN-2 fwd/fwd+bwd tokens/s (H=16,d=128,T=4K); decode steps/s; % of roofline"
CHUNK = 64


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ peaks / roofline
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def fwd_bytes(B, T, H, D):
    """Algorithmic bytes of one forward: per token-head q,k,v,b,w (bf16) + log alpha (fp32)
    read and o (bf16) written = 2048 B at D=128; plus S0 read and S_T written (fp32)."""
    per_tok_head = 5 * 2 * D + 4 * D + 2 * D
    return B * T * H * per_tok_head + B * H * 2 * D * D * 4


def bwd_bytes(B, T, H, D):
    """Per token-head: q,k,v,b,w,do read and dq,dk,dv,db,dw written (bf16), log alpha read
    and its gradient written (fp32); plus S0 read and dS0 written (dS_T = 0 is not read)."""
    per_tok_head = 11 * 2 * D + 2 * 4 * D
    return B * T * H * per_tok_head + B * H * 2 * D * D * 4


def decode_bytes(N, H, D):
    """State read + written (fp32), q,k,v,b,w read and o written (bf16), log alpha (fp32)."""
    return N * H * (2 * D * D * 4 + 6 * 2 * D + 4 * D)


def fwd_flops(B, T, H, D, C=CHUNK):
    """Dense-tile flops per token-head: 5 C x C x d products (A, W, U, P, P U~) and
    3 C x d x d products (W S, Q~ S, K^^T U~) per chunk = 10 C d + 6 d^2."""
    return B * T * H * (10 * C * D + 6 * D * D)


def device_code_sha(text: str, kernel_def: str):
    """SHA-256 of a kernel source file's text up to the closing brace of the kernel's
    definition: the device code the kernel is built from (constants, helpers and the kernel
    itself), without the host code after it."""
    i = text.index(kernel_def)
    j = text.index("\n}\n", i) + 3
    return hashlib.sha256(text[:j].encode()).hexdigest()


def _code_matches(src_name: str, kernel_def: str, sha: str) -> bool:
    src = os.path.join(ROOT, "gated_delta_rule_78_b200", "csrc", src_name)
    if not os.path.exists(src):
        return False
    try:
        return device_code_sha(open(src).read(), kernel_def) == sha
    except ValueError:
        return False


def kernel_traffic(kernel_src: str):
    """DRAM bytes per launch (or per call, for a record that spans several kernels) from the
    committed ncu summary, if it was taken on the current device code of every kernel it covers
    (same SHA-256 of each file up to the kernel's end), else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(kernel_src)
    if not e:
        return None
    if "kernels" in e:  # several kernels: every one must still be the captured code
        ok = all(_code_matches(k["file"], k["kernel_def"], k["sha256_device"]) for k in e["kernels"])
        return e.get("bytes_per_call") if ok else None
    try:
        ok = _code_matches(kernel_src, e["kernel_def"], e["sha256_device"])
    except KeyError:
        return None
    return e.get("bytes_per_launch") if ok else None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        self.dev = device_index

    def _gpu_id(self):
        try:
            u = str(torch.cuda.get_device_properties(self.dev).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return str(self.dev)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self._gpu_id()],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines += [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        busy = [x for x in sm if x > 0.5 * (smax or max(sm))] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ timing helpers
def time_region(fn, steps, warmup, stream):
    for _ in range(warmup):
        fn()
    stream.synchronize()
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1))


# ------------------------------------------------------------------ multi-rank plumbing
def max_over_ranks(ms: float) -> float:
    """The slowest rank's time: every rank joins the same all-reduce (MAX), then a barrier.
    The tensor lives where the process group's backend wants it (cuda for nccl, cpu for gloo)."""
    if not torch.distributed.is_initialized():
        return ms
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.barrier()
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch of the workload (weak scaling, no data-path collective)."""
    return 1234 + rank


def job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


def roofline(bytes_per_launch, ms_per_launch, pk, traffic=None, bound="hbm"):
    achieved = bytes_per_launch / (ms_per_launch * 1e-3) / 1e9
    return {"bound": bound, "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
            "algorithmic_bytes": bytes_per_launch, "peak_source": pk["source"] + " (burst copy)"}


# ------------------------------------------------------------------ CPU oracle baseline
def cpu_baseline(w, target_s=12.0, seed=0):
    """Time the fp64 oracle forward on a bounded sample of (batch, head) sequences of the
    workload (full length T), sized for about `target_s` seconds of host work."""
    import oracle  # test infrastructure: only this leg of the benchmark runs it
    cores = oracle.default_threads()
    T, D = w["T"], w["Dk"]
    one = make_inputs(1, T, 1, D, D, dtype=w["dtype"], seed=seed)
    t0 = time.perf_counter()
    oracle.ref_fwd(one["q"], one["k"], one["v"], one["log_alpha"], one["b"], one["w"], one["S0"], nthreads=1)
    per_seq = time.perf_counter() - t0
    # as many full-length sequences of the workload's shape as fit about target_s seconds
    nseq = max(cores, int(target_s * cores / max(per_seq, 1e-3)))
    nseq = min((nseq // cores) * cores or cores, 64 * cores)
    x = make_inputs(1, T, nseq, D, D, dtype=w["dtype"], seed=seed + 1)
    t0 = time.perf_counter()
    oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], nthreads=cores)
    dt = time.perf_counter() - t0
    tokens = nseq * T / w["H"]  # a token covers all H heads
    return {"value": round(tokens / dt, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 token-recurrence forward of {nseq} (batch, head) sequences of "
                      f"T={T}, d={D} ({nseq / w['H']:.2f} batch rows of H={w['H']}), {dt:.1f} s"}


def run_reference(args):
    """--impl reference: the fp64 oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = dict(WORKLOADS[args.workload])
    cores = oracle.default_threads()
    T, D, H = w["T"], w["Dk"], w["H"]
    # one step = one batch row of the workload (all H heads, full length T)
    x = make_inputs(1, T, H, D, D, dtype=w["dtype"], seed=0)
    arg = (x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    for _ in range(args.warmup):
        oracle.ref_fwd(*arg, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.ref_fwd(*arg, nthreads=cores)
    dt = time.perf_counter() - t0
    value = args.steps * T / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B_per_step": 1, "T": T, "H": H, "d": D,
                       "note": "each step is one batch row (all heads) of the workload"},
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} steps x 1 batch row (H={H}, T={T}, d={D})"},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import gated_delta_rule_78_b200 as g
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    g.load()
    stream = torch.cuda.current_stream()
    pk = peaks()
    w = dict(WORKLOADS[args.workload])
    B, T, H, D = w["B"], w["T"], w["H"], w["Dk"]
    tokens = B * T  # per rank
    clocks = ClockSampler(dev.index)

    if args.only in ("prologue", "scan"):
        run_part(args, g, w, dev, stream, rank, world, pk)
        return

    # ---- forward (headline)
    x = make_inputs(B, T, H, D, D, dtype=w["dtype"], seed=rank_seed(rank), device=str(dev), with_do=True)
    o = torch.empty_like(x["v"])
    ST = torch.empty_like(x["S0"])

    def fwd():
        g.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], o=o, S_T=ST)

    parts = {"fwd", "bwd", "decode"} if not args.only else {args.only}
    if args.fwd_only:
        parts = {"fwd"}
    clocks.start()
    fb = fwd_bytes(B, T, H, D)
    ms_fwd = None
    if "fwd" in parts:
        ms_fwd = time_region(fwd, args.steps, args.warmup, stream) / args.steps
        assert g.gdn2_sync_status() == 0, "a kernel reported a timeout"

    # ---- forward + backward on the same batch
    extras = {}
    if "bwd" in parts:
        nws = g.gdn2_workspace_size(1, x["q"].dtype, B, T, H, D, D)
        ws = torch.empty(nws, dtype=torch.uint8, device=dev)
        grads = {"dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"]),
                 "dlog_alpha": torch.empty_like(x["log_alpha"]), "db": torch.empty_like(x["b"]),
                 "dw": torch.empty_like(x["w"]), "dS0": torch.empty_like(x["S0"])}

        def bwd():
            g.gdn2_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"],
                             None, workspace=ws, out=grads)

        ksteps = max(3, args.steps // 4)
        ms_bwd = time_region(bwd, ksteps, max(3, args.warmup // 2), stream) / ksteps
        assert g.gdn2_sync_status() == 0
        bb = bwd_bytes(B, T, H, D)
        extras["fwd_bwd"] = {"bwd_ms": round(ms_bwd, 4), "steps": ksteps,
                             "bwd_roofline": roofline(bb, ms_bwd, pk, kernel_traffic("backward") if args.workload == "layer_4k" else None),
                             "bwd_launches": 1 + 3}
        if ms_fwd is not None:
            # a training step: the forward records the chunk-boundary states and chunk factors into
            # the backward's workspace, and the backward skips its own states pass
            o_tr = torch.empty_like(x["v"])
            S_tr = torch.empty_like(x["S0"])

            def train_step():
                g.gdn2_chunk_fwd_save(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], workspace=ws,
                                      o=o_tr, S_T=S_tr)
                g.gdn2_chunk_bwd_saved(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"],
                                       None, workspace=ws, out=grads)

            ms_fb = time_region(train_step, ksteps, max(3, args.warmup // 2), stream) / ksteps
            assert g.gdn2_sync_status() == 0
            extras["fwd_bwd"].update({
                "step": "gdn2_chunk_fwd_save + gdn2_chunk_bwd_saved", "launches_per_step": 1 + 3,
                "value": round(job_rate(tokens, world, ms_fb), 1), "unit": "tokens/s",
                "ms_per_step": round(ms_fb, 4), "roofline": roofline(fb + bb, ms_fb, pk),
                "fwd_plus_standalone_bwd_ms": round(ms_fwd + ms_bwd, 4)})
            del o_tr, S_tr
        del ws, grads

    if "decode" in parts:
        # ---- decode: 256 sequences, 1024 steps, per-step inputs resident
        dw = DECODE_WORKLOAD
        N, Hd, Dd, nsteps = dw["N"], dw["H"], dw["Dk"], dw["steps"]
        ds = DecodeStream(N, Hd, Dd, Dd, dtype=dw["dtype"], seed=99 + rank, device=str(dev))
        S = ds.S0
        steps_in = [ds.step() for _ in range(nsteps)]
        od = torch.empty(N, Hd, Dd, dtype=torch.bfloat16, device=dev)
        it = {"i": 0}

        def dec():
            s = steps_in[it["i"] % nsteps]
            it["i"] += 1
            g.gdn2_decode_step(s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"], S, o=od)

        ms_all = time_region(dec, nsteps, 16, stream)
        assert g.gdn2_sync_status() == 0
        ms_dec = ms_all / nsteps
        extras["decode"] = {
            "value": round(world * 1e3 / ms_dec, 1), "unit": "steps/s",
            "tokens_per_s": round(world * N * 1e3 / ms_dec, 1), "us_per_step": round(ms_dec * 1e3, 3),
            "steps": nsteps, "workload": f"N={N}, H={Hd}, d={Dd}, fp32 state in place",
            "roofline": roofline(decode_bytes(N, Hd, Dd), ms_dec, pk, kernel_traffic("decode.cu")),
            "launches_per_step": 1}
        del steps_in
    if "fwd" in parts and not args.no_sweep:
        # ---- variable length: the same 32,768 tokens as the headline, as 16 packed sequences whose
        #      lengths are log-uniform in [256, 8192] (seeded), forward and backward
        rng = np.random.default_rng(7)
        lens = np.exp(rng.uniform(np.log(256), np.log(8192), 16))
        lens = np.maximum(1, np.round(lens / lens.sum() * tokens)).astype(np.int64)
        lens[-1] += tokens - lens.sum()
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
        xv = make_inputs(1, tokens, H, D, D, dtype=w["dtype"], seed=rank_seed(rank) + 17, device=str(dev), with_do=True)
        S0v = torch.zeros(len(lens), H, D, D, device=dev)
        ov = torch.empty_like(xv["v"][0])
        Sv = torch.empty_like(S0v)

        def fwd_v():
            g.gdn2_chunk_fwd_varlen(xv["q"], xv["k"], xv["v"], xv["log_alpha"], xv["b"], xv["w"], cu, S0v, o=ov, S_T=Sv)

        ms_v = time_region(fwd_v, 10, 3, stream) / 10
        wsv = torch.empty(g.gdn2_workspace_size(3, xv["q"].dtype, len(lens), tokens, H, D, D), dtype=torch.uint8,
                          device=dev)

        def bwd_v():
            g.gdn2_chunk_bwd_varlen(xv["q"], xv["k"], xv["v"], xv["log_alpha"], xv["b"], xv["w"], cu, S0v, xv["do"],
                                    workspace=wsv)

        ms_vb = time_region(bwd_v, 5, 3, stream) / 5
        assert g.gdn2_sync_status() == 0
        # ---- scalar decay (one log alpha per token and head, Gated DeltaNet style), per-channel b, w:
        #      the tensor-core forward computes one exponential pair per token instead of per channel
        gsc = -torch.nn.functional.softplus(
            torch.randn(B, T, H, generator=torch.Generator(device=str(dev)).manual_seed(5), device=dev) - 3.0)
        wsg = torch.empty(max(16, g.gdn2_workspace_size_gated(0, g.DECAY_SCALAR, x["q"].dtype, B, T, H, D, D)),
                          dtype=torch.uint8, device=dev)

        def fwd_sd():
            g.gdn2_chunk_fwd_gated(x["q"], x["k"], x["v"], gsc, x["b"], x["w"], x["S0"], flags=g.DECAY_SCALAR, o=o,
                                   S_T=ST, workspace=wsg)

        ms_sd = time_region(fwd_sd, 20, 3, stream) / 20
        assert g.gdn2_sync_status() == 0
        sd_bytes = fwd_bytes(B, T, H, D) - B * T * H * (4 * D - 4)
        extras["scalar_decay"] = {"workload": f"B={B}, T={T}, H={H}, d={D}; log alpha [B,T,H], b and w per channel",
                                  "ms": round(ms_sd, 4), "tokens_per_s": round(job_rate(tokens, world, ms_sd), 1),
                                  "algorithmic_bytes": sd_bytes,
                                  "hbm_frac": round(sd_bytes / (ms_sd * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        del wsg
        # ---- KDA and Gated DeltaNet shapes: b = w = beta, one value per (token, head), with the
        #      per-channel decay (KDA) or a scalar one (Gated DeltaNet); the tensor-core forward
        #      reads the gates as they are
        beta = torch.sigmoid(torch.randn(B, T, H, generator=torch.Generator(device=str(dev)).manual_seed(6),
                                         device=dev)).to(x["q"].dtype)
        gate_pts = {}
        for name, fl, gdec in (("kda", g.ERASE_SCALAR | g.WRITE_SCALAR, x["log_alpha"]),
                               ("gated_deltanet", g.ERASE_SCALAR | g.WRITE_SCALAR | g.DECAY_SCALAR, gsc)):
            wsk = torch.empty(max(16, g.gdn2_workspace_size_gated(0, fl, x["q"].dtype, B, T, H, D, D)),
                              dtype=torch.uint8, device=dev)

            def fwd_k():
                g.gdn2_chunk_fwd_gated(x["q"], x["k"], x["v"], gdec, beta, beta, x["S0"], flags=fl, o=o, S_T=ST,
                                       workspace=wsk)

            ms_k = time_region(fwd_k, 20, 3, stream) / 20
            assert g.gdn2_sync_status() == 0
            kb = fwd_bytes(B, T, H, D) - B * T * H * 2 * (2 * D - 2) - (B * T * H * (4 * D - 4) if gdec is gsc else 0)
            # its backward: the scalar gates (b, w and, for Gated DeltaNet, the decay) run natively
            wsb = torch.empty(g.gdn2_workspace_size_gated(1, fl, x["q"].dtype, B, T, H, D, D), dtype=torch.uint8,
                              device=dev)
            grk = {"dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"]),
                   "dlog_alpha": torch.empty_like(gdec), "db": torch.empty_like(beta), "dw": torch.empty_like(beta),
                   "dS0": torch.empty_like(x["S0"])}

            def bwd_k():
                g.gdn2_chunk_bwd_gated(x["q"], x["k"], x["v"], gdec, beta, beta, x["S0"], x["do"], flags=fl,
                                       workspace=wsb, out=grk)

            ms_kb = time_region(bwd_k, 5, 3, stream) / 5
            assert g.gdn2_sync_status() == 0
            del wsb, grk
            gate_pts[name] = {"workload": f"B={B}, T={T}, H={H}, d={D}; b = w = beta [B,T,H]" +
                              ("; log alpha [B,T,H]" if gdec is gsc else "; log alpha per channel"),
                              "ms": round(ms_k, 4), "tokens_per_s": round(job_rate(tokens, world, ms_k), 1),
                              "algorithmic_bytes": kb, "hbm_frac": round(kb / (ms_k * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                              "workspace_bytes": int(wsk.numel()) if wsk.numel() > 16 else 0,
                              "bwd_ms": round(ms_kb, 4)}
            del wsk
        extras.update(gate_pts)
        # ---- input prologue fused in the chunk kernel, against a separate pass + the plain forward
        xr = make_inputs(B, T, H, D, D, dtype=w["dtype"], seed=rank_seed(rank) + 31, device=str(dev), raw=True)
        pro_flags = g.QK_L2NORM | g.BW_LOGITS
        pro_out = {n: torch.empty_like(xr[n]) for n in ("q", "k", "b", "w")}

        def fwd_pro():
            g.gdn2_chunk_fwd_gated(xr["q"], xr["k"], xr["v"], xr["log_alpha"], xr["b"], xr["w"], xr["S0"],
                                   flags=pro_flags, o=o, S_T=ST)

        def fwd_unfused():
            g.gdn2_prologue(xr["q"], xr["k"], xr["b"], xr["w"], flags=pro_flags, out=pro_out)
            g.gdn2_chunk_fwd(pro_out["q"], pro_out["k"], xr["v"], xr["log_alpha"], pro_out["b"], pro_out["w"], xr["S0"],
                             o=o, S_T=ST)

        ms_pro = time_region(fwd_pro, 20, 3, stream) / 20
        ms_unf = time_region(fwd_unfused, 20, 3, stream) / 20
        assert g.gdn2_sync_status() == 0
        fb_pro = fwd_bytes(B, T, H, D)
        extras["prologue"] = {"workload": f"B={B}, T={T}, H={H}, d={D}; raw q, k and b, w logits",
                              "fused_ms": round(ms_pro, 4), "unfused_ms": round(ms_unf, 4),
                              "fused_tokens_per_s": round(job_rate(tokens, world, ms_pro), 1),
                              "algorithmic_bytes": fb_pro,
                              "fused_hbm_frac": round(fb_pro / (ms_pro * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                              "unfused_extra_bytes": 8 * B * T * H * D * xr["q"].element_size()}
        del xr, pro_out
        # ---- head size 64 (same model width: H = 32), bf16, on the tensor-core forward
        x64 = make_inputs(B, T, 2 * H, D // 2, D // 2, dtype=w["dtype"], seed=rank_seed(rank) + 29, device=str(dev),
                          with_do=True)
        o64 = torch.empty_like(x64["v"])
        S64 = torch.empty_like(x64["S0"])

        def fwd_64():
            g.gdn2_chunk_fwd(x64["q"], x64["k"], x64["v"], x64["log_alpha"], x64["b"], x64["w"], x64["S0"], o=o64,
                             S_T=S64)

        ms_64 = time_region(fwd_64, 10, 3, stream) / 10
        assert g.gdn2_sync_status() == 0
        b64 = fwd_bytes(B, T, 2 * H, D // 2)
        # its backward, with the same workspace rules as the headline one
        ws64 = torch.empty(g.gdn2_workspace_size(1, x64["q"].dtype, B, T, 2 * H, D // 2, D // 2), dtype=torch.uint8,
                           device=dev)
        gr64 = {"dq": torch.empty_like(x64["q"]), "dk": torch.empty_like(x64["k"]), "dv": torch.empty_like(x64["v"]),
                "dlog_alpha": torch.empty_like(x64["log_alpha"]), "db": torch.empty_like(x64["b"]),
                "dw": torch.empty_like(x64["w"]), "dS0": torch.empty_like(x64["S0"])}

        def bwd_64():
            g.gdn2_chunk_bwd(x64["q"], x64["k"], x64["v"], x64["log_alpha"], x64["b"], x64["w"], x64["S0"], x64["do"],
                             None, workspace=ws64, out=gr64)

        ms_64b = time_region(bwd_64, 5, 3, stream) / 5
        assert g.gdn2_sync_status() == 0
        bb64 = bwd_bytes(B, T, 2 * H, D // 2)
        extras["d64"] = {"workload": f"B={B}, T={T}, H={2 * H}, d={D // 2}, bf16", "ms": round(ms_64, 4),
                         "tokens_per_s": round(job_rate(tokens, world, ms_64), 1), "algorithmic_bytes": b64,
                         "hbm_frac": round(b64 / (ms_64 * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                         "bwd_ms": round(ms_64b, 4), "bwd_algorithmic_bytes": bb64,
                         "bwd_hbm_frac": round(bb64 / (ms_64b * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        del x64, o64, S64, ws64, gr64
        extras["varlen"] = {"sequences": len(lens), "lengths": [int(v) for v in lens], "tokens": tokens,
                            "fwd_ms": round(ms_v, 4), "fwd_tokens_per_s": round(job_rate(tokens, world, ms_v), 1),
                            "fwd_hbm_frac": round(fwd_bytes(1, tokens, H, D) / (ms_v * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                            "bwd_ms": round(ms_vb, 4)}
        del xv, ov, Sv, wsv

        # ---- sequence-length sweep at a fixed 65,536 tokens per call (one forward per step)
        sweep = {}
        for name in ("sweep_2k", "sweep_4k", "sweep_8k", "sweep_16k", "sweep_32k"):
            sw = WORKLOADS[name]
            xs = make_inputs(sw["B"], sw["T"], sw["H"], sw["Dk"], sw["Dv"], dtype=sw["dtype"], seed=rank_seed(rank),
                             device=str(dev))
            os_ = torch.empty_like(xs["v"])
            Ss = torch.empty_like(xs["S0"])
            # few long chains take the chunk-parallel scan, which needs a workspace
            nws = g.gdn2_workspace_size(0, xs["q"].dtype, sw["B"], sw["T"], sw["H"], sw["Dk"], sw["Dv"])
            wss = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)

            def fwd_s():
                g.gdn2_chunk_fwd(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["b"], xs["w"], xs["S0"], o=os_, S_T=Ss,
                                 workspace=wss)

            ks = 10
            ms_s = time_region(fwd_s, ks, 3, stream) / ks
            assert g.gdn2_sync_status() == 0
            bs = fwd_bytes(sw["B"], sw["T"], sw["H"], sw["Dk"])
            sweep[name] = {"T": sw["T"], "B": sw["B"], "ctas": sw["B"] * sw["H"], "scan": nws > 0, "ms": round(ms_s, 4),
                           "tokens_per_s": round(job_rate(sw["B"] * sw["T"], world, ms_s), 1),
                           "hbm_frac": round(bs / (ms_s * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
            del xs, os_, Ss, wss
        extras["sweep"] = sweep
    clocks.stop()
    if ms_fwd is None:
        # a single non-forward part was asked for (profiling runs): report it alone
        if rank == 0:
            print(json.dumps({"metric": METRIC, "only": args.only, "steps": args.steps,
                              "warmup": args.warmup, "config": {"workload": args.workload},
                              **extras}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    value = job_rate(tokens, world, ms_fwd)

    # ---- end to end through the C-ABI call with host buffers (gdn2_chunk_fwd_host: the copies in,
    #      the kernels and the copies out pipelined by batch rows inside the call)
    hx = {n: t.to("cpu").pin_memory() for n, t in x.items() if n != "do"}
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hS = torch.empty(ST.shape, dtype=ST.dtype, pin_memory=True)
    wsh = torch.empty(max(16, g.gdn2_workspace_size(4, x["q"].dtype, B, T, H, D, D)), dtype=torch.uint8, device=dev)

    def e2e():
        g.gdn2_chunk_fwd_host(hx["q"], hx["k"], hx["v"], hx["log_alpha"], hx["b"], hx["w"], hx["S0"], o=ho, S_T=hS,
                              workspace=wsh)

    ke = max(3, args.steps // 4)
    ms_e2e = time_region(e2e, ke, 2, stream) / ke
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = o.numel() * o.element_size() + ST.numel() * ST.element_size()

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_fwd, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "T": T, "H": H, "d_k": D, "d_v": D, "chunk": CHUNK,
                   "inputs": "bf16 q,k,v,b,w; fp32 log alpha and state; S0 ~ N(0, 0.02)",
                   "l2": f"inputs exceed L2 ({fb / 1e9:.2f} GB per step vs 126 MB): no flush",
                   "parallelism": f"dp{world}: independent (batch, head) sequences per rank, no collective"},
        "e2e": {"value": round(job_rate(tokens, world, ms_e2e), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 3)},
        "gpu_launches": args.steps,
        "roofline": roofline(fb, ms_fwd, pk, kernel_traffic("fwd_tc.cu")),
        "flops_per_step": fwd_flops(B, T, H, D),
        "tensor_frac": round(fwd_flops(B, T, H, D) / (ms_fwd * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
        "clocks": clocks.summary(),
    }
    line.update(extras)
    if world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_part(args, g, w, dev, stream, rank, world, pk):
    """One extra measured alone, for profiling runs: `prologue` (layer_4k with raw q, k and gate
    logits: the fused forward, then the separate pass + plain forward) or `scan` (B=2, T=32768,
    H=16: the chunk-parallel scan, then the serial chain)."""
    out = {"metric": METRIC, "only": args.only, "steps": args.steps, "warmup": args.warmup}
    if args.only == "prologue":
        B, T, H, D = w["B"], w["T"], w["H"], w["Dk"]
        xr = make_inputs(B, T, H, D, D, dtype=w["dtype"], seed=rank_seed(rank) + 31, device=str(dev), raw=True)
        o = torch.empty_like(xr["v"])
        ST = torch.empty_like(xr["S0"])
        flags = g.QK_L2NORM | g.BW_LOGITS
        pro = {n: torch.empty_like(xr[n]) for n in ("q", "k", "b", "w")}

        def fused():
            g.gdn2_chunk_fwd_gated(xr["q"], xr["k"], xr["v"], xr["log_alpha"], xr["b"], xr["w"], xr["S0"],
                                   flags=flags, o=o, S_T=ST)

        def unfused():
            g.gdn2_prologue(xr["q"], xr["k"], xr["b"], xr["w"], flags=flags, out=pro)
            g.gdn2_chunk_fwd(pro["q"], pro["k"], xr["v"], xr["log_alpha"], pro["b"], pro["w"], xr["S0"], o=o, S_T=ST)

        out["fused_ms"] = round(time_region(fused, args.steps, args.warmup, stream) / args.steps, 4)
        out["unfused_ms"] = round(time_region(unfused, args.steps, args.warmup, stream) / args.steps, 4)
        out["config"] = {"workload": f"{args.workload}, raw q, k and b, w logits"}
    else:
        sw = WORKLOADS["sweep_32k"]
        B, T, H, D = sw["B"], sw["T"], sw["H"], sw["Dk"]
        xs = make_inputs(B, T, H, D, D, dtype=sw["dtype"], seed=rank_seed(rank), device=str(dev))
        o = torch.empty_like(xs["v"])
        ST = torch.empty_like(xs["S0"])
        nws = g.gdn2_workspace_size(0, xs["q"].dtype, B, T, H, D, D)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
        none = torch.empty(16, dtype=torch.uint8, device=dev)

        def run(wsp):
            return lambda: g.gdn2_chunk_fwd(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["b"], xs["w"], xs["S0"],
                                            o=o, S_T=ST, workspace=wsp)

        out["scan_ms"] = round(time_region(run(ws), args.steps, args.warmup, stream) / args.steps, 4)
        out["serial_ms"] = round(time_region(run(none), args.steps, args.warmup, stream) / args.steps, 4)
        out["config"] = {"workload": "sweep_32k", "B": B, "T": T, "H": H, "chains": B * H, "workspace": nws}
    assert g.gdn2_sync_status() == 0
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="layer_4k", choices=sorted(WORKLOADS))
    ap.add_argument("--fwd-only", action="store_true", help="skip the fwd+bwd and decode figures")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-sweep", action="store_true", help="skip the sequence-length sweep")
    ap.add_argument("--only", choices=["fwd", "bwd", "decode", "prologue", "scan"], default=None,
                    help="time one part only (for profiling runs): the headline forward, the backward, "
                         "decode, the fused input prologue against a separate pass, or the chunk-parallel "
                         "scan against the serial chain at B=2, T=32K")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    args.steps = max(1, args.steps)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
