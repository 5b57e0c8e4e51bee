"""Benchmark of the gated-retention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python -m torch.distributed.run --nproc-per-node N bench.py --gpus N ...   (N > 1)

One step = one chunkwise prefill of one gated-retention layer of the 3B shape (batch 1,
24 heads, 32768 tokens, d_k = d_v = 128, bf16 inputs, fp32 state, g ~ N(2, 1), tau = 16) through
the C ABI, inputs resident in HBM.  The printed JSON line carries:
  value     whole-job prefill throughput (Mtok/s; every rank runs its own sequence: weak scaling)
  roofline  the prefill kernel against measured HBM bandwidth (1028 algorithmic bytes per
            token and head: q, k, v, o in bf16 plus the fp32 gate logit)
  decode    batched decode at batch 64 (state of 64 x 24 x 128 x 128 fp32 from a 4096-token
            prefill, 256 steps), tok/s and its HBM roofline
  e2e       the same prefill metric with host buffers: pinned host -> device copies of q, k, v, g
            and device -> host copies of o and the final state inside the timed region
  varlen_epilogue  8 packed sequences of seeded lengths in [1024, 65536] with harsher gates
            (g ~ N(0, 2)): varlen prefill, then the per-head GroupNorm * swish(X W_G) epilogue
            (X [T, 3072], W_G [3072, 3072]); Mtok/s of the pair, and the epilogue GEMM against
            the measured bf16 tensor peak
  cpu_baseline  the fp64 CPU oracle on the same workload (rank 0 only)
With --impl reference the oracle alone is timed, on host cores, as the reference arm.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gRet prefill Mtok/s (H=24,d=128,N=32K); decode tok/s @bs64; % of roofline"
B, N, H, D = 1, 32768, 24, 128
BYTES_PER_TOKEN_HEAD = 4 * D * 2 + 4          # q, k, v, o (bf16) + g (fp32)
DEC_B, DEC_PREFILL, DEC_STEPS = 64, 4096, 256
DEC_BYTES_PER_HEAD = 2 * D * D * 4 + 4 * D * 2 + 4   # state read + write, q k v o, g
WORKLOAD = ("gRet chunkwise prefill, batch 1, H=24, N=32768, d_k=d_v=128, bf16 q/k/v "
            "~N(0,1)/sqrt(128), g~N(2,1), tau=16, fp32 state")


def bench_config(world):
    """The workload description printed by both arms."""
    return {"workload": WORKLOAD, "tokens_per_rank": B * N, "heads": H, "d": D,
            "parallelism": "independent sequence per GPU" if world > 1 else "1 GPU",
            "l2": "inputs and outputs (808 MB per step) larger than L2 (126 MB); "
                  "L2 not flushed"}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def measured_tensor_peak():
    """bf16 dense TFLOP/s: the burst figure (a kernel timed on its own)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    rank, world = 0, 1
    if n_gpus > 1 or "WORLD_SIZE" in os.environ:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        local = int(os.environ.get("LOCAL_RANK", str(rank)))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a host float over all ranks (the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base, rank):
    """Seed of a rank's own synthetic sequence: every rank processes different data."""
    return base + 1000 * rank


def kernel_code_digest(path):
    """sha256 (16 hex digits) of a CUDA source with its comments and whitespace removed, so that
    a measurement taken on the code stays valid across comment-only edits."""
    import hashlib
    import re
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    src = re.sub(r"\s+", " ", src).strip()
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def traffic_from_profile(src_name, summary_name, units=None):
    """DRAM bytes per launch of a kernel from its committed ncu summary under profiles/, if that
    summary was taken on the current code of csrc/<src_name> (else None).  A summary taken on a
    smaller case states its `units` (tokens); the bytes are then scaled to `units` of this run,
    the traffic of these kernels growing in proportion to the tokens they process."""
    src = os.path.join(ROOT, "gated_retention_linear_b200", "csrc", src_name)
    summ = os.path.join(ROOT, "profiles", summary_name)
    try:
        kv = {}
        for line in open(summ):
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        digest = kv.get("kernel_code_sha256_16", "").split()
        if digest and digest[0] == kernel_code_digest(src):
            b = float(kv["dram_bytes_per_launch"].split()[0])
            if units is not None and "profile_units" in kv:
                b *= units / float(kv["profile_units"].split()[0])
            return int(b)
    except Exception:
        pass
    return None


def prefill_traffic_from_profile():
    return traffic_from_profile("prefill_tc.cu", "prefill_tc_kernel_32k.txt")


def run_gpu(args):
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI

    rank, world = dist_setup(args.gpus)
    dev = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    hbm_peak, peak_kind = measured_peaks()

    # ---------------- prefill, inputs resident in HBM
    inp = SI.gret_inputs(B, N, H, D, dtype=torch.bfloat16, g_mean=2.0, g_std=1.0,
                         seed=rank_seed(2, rank), device="cuda")
    q, k, v, g = inp["q"], inp["k"], inp["v"], inp["g"]
    o = torch.empty_like(v)
    s_out = torch.empty((B, H, D, D), dtype=torch.float32, device="cuda")
    need = G.gret_prefill_workspace_size(torch.bfloat16, B * N, B, H, D, D, 0)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    def step():
        G.gret_prefill_chunkwise(q, k, v, g, state_out=s_out, o=o, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if G.gret_workspace_status(ws) != 0:
        raise RuntimeError("prefill reported a timed-out wait during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_total = t0.elapsed_time(t1)
    launch_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    ms_total = max_over_ranks(ms_total, world)
    if G.gret_workspace_status(ws) != 0:
        raise RuntimeError("prefill reported a timed-out wait")
    ms_per_step = ms_total / args.steps
    tokens_all = B * N * world * args.steps
    value = tokens_all / (ms_total * 1e-3) / 1e6
    alg_bytes = B * N * H * BYTES_PER_TOKEN_HEAD
    achieved = alg_bytes / (launch_ms * 1e-3) / 1e9

    # ---------------- the same prefill at every chunk size the library takes
    sweep = None
    if args.chunk_sweep:
        sweep = {}
        for ch in (16, 32, 64, 128):
            def stepc():
                G.gret_prefill_chunkwise(q, k, v, g, state_out=s_out, o=o, workspace=ws, chunk=ch)
            for _ in range(2):
                stepc()
            torch.cuda.synchronize()
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            nrep = 3 if ch < 128 else 10
            c0.record(stream)
            for _ in range(nrep):
                stepc()
            c1.record(stream)
            torch.cuda.synchronize()
            cms = c0.elapsed_time(c1) / nrep
            sweep[str(ch)] = {"ms": cms, "Mtok_s": B * N / (cms * 1e-3) / 1e6,
                              "hbm_frac": alg_bytes / (cms * 1e-3) / 1e9 / hbm_peak,
                              "path": "tcgen05" if ch == 128 else "CUDA cores (fp32 FMA)"}

    # ---------------- decode at batch 64
    dec = None
    if not args.no_decode:
        dinp = SI.gret_inputs(DEC_B, DEC_PREFILL, H, D, dtype=torch.bfloat16,
                              seed=rank_seed(4, rank),
                              device="cuda")
        _, state = G.gret_prefill_chunkwise(dinp["q"], dinp["k"], dinp["v"], dinp["g"],
                                            state_out=True)
        del dinp
        steps_in = SI.gret_inputs(DEC_B, DEC_STEPS, H, D, dtype=torch.bfloat16,
                                  seed=rank_seed(40, rank), device="cuda")
        qs = steps_in["q"].permute(1, 0, 2, 3).contiguous()    # [steps, B, H, d]
        ks = steps_in["k"].permute(1, 0, 2, 3).contiguous()
        vs = steps_in["v"].permute(1, 0, 2, 3).contiguous()
        gs = steps_in["g"].permute(1, 0, 2).contiguous()
        od = torch.empty((DEC_B, H, D), dtype=torch.bfloat16, device="cuda")
        state0 = state.clone()
        for w in range(args.warmup):
            G.gret_decode_step(qs[w], ks[w], vs[w], gs[w], state, o=od)
        state.copy_(state0)
        torch.cuda.synchronize()
        barrier(world)
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for s in range(DEC_STEPS):
            G.gret_decode_step(qs[s], ks[s], vs[s], gs[s], state, o=od)
        d1.record(stream)
        torch.cuda.synchronize()
        eager_ms = max_over_ranks(d0.elapsed_time(d1), world)
        # the same 256 launches captured once in a CUDA graph and replayed, as a serving loop
        # runs them: no host work and no launch gaps between the steps
        state.copy_(state0)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for s in range(DEC_STEPS):
                G.gret_decode_step(qs[s], ks[s], vs[s], gs[s], state, o=od)
        state.copy_(state0)
        graph.replay()                     # one untimed replay (the graph's first upload)
        state.copy_(state0)
        torch.cuda.synchronize()
        barrier(world)
        d0.record(stream)
        graph.replay()
        d1.record(stream)
        torch.cuda.synchronize()
        dms = max_over_ranks(d0.elapsed_time(d1), world)
        del graph
        dec_bytes = DEC_B * H * DEC_BYTES_PER_HEAD
        dec_ach = dec_bytes / (dms / DEC_STEPS * 1e-3) / 1e9
        dec = {"value": DEC_B * DEC_STEPS * world / (dms * 1e-3), "unit": "tok/s",
               "ms_per_step": dms / DEC_STEPS, "steps": DEC_STEPS, "batch": DEC_B,
               "gpu_launches": DEC_STEPS, "launch": "CUDA graph of the 256 steps",
               "eager": {"value": DEC_B * DEC_STEPS * world / (eager_ms * 1e-3),
                         "ms_per_step": eager_ms / DEC_STEPS,
                         "launch": "one ABI call per step from Python"},
               "roofline": {"bound": "hbm", "achieved": dec_ach, "peak": hbm_peak,
                            "unit": "GB/s", "frac": dec_ach / hbm_peak,
                            "peak_kind": peak_kind,
                            "traffic": traffic_from_profile("decode.cu", "decode_kernel_bs64.txt")},
               "l2": "state (201 MB) larger than L2 (126 MB); not flushed between steps"}
        del qs, ks, vs, gs, state, state0

    # The legs whose kernels are memory- or latency-bound run before the two with dense GEMMs
    # (the varlen epilogue and the layer): those hold the GPU at its power cap, and the clocks
    # that follow them stay lowered for a while (measured: the sliding-window and per-channel
    # legs 12-35 % slower when run after them).

    # ---------------- per-key-channel gate variant of the prefill, same 3B shapes
    ew = None
    if not args.no_elementwise:
        ew = run_elementwise(args, rank, world, stream, ms_per_step)

    # ---------------- sliding-window attention, the other Self-Decoder mixer, same shapes
    swa = None
    if not args.no_swa:
        swa = run_swa(args, rank, world, stream, ms_per_step)

    # ---------------- the long-context prefill: one 524288-token sequence, 24 heads
    long_ctx = None
    if not args.no_long:
        long_ctx = run_long_context(args, rank, world, stream, hbm_peak, peak_kind)

    # ---------------- varlen prefill + GroupNorm * swish(X W_G) epilogue
    epi = None
    if not args.no_epilogue:
        epi = run_varlen_epilogue(args, rank, world, stream, hbm_peak)

    # ---------------- one mixer layer: projection GEMM -> prefill -> GroupNorm * gate
    lay = None
    if not args.no_layer:
        lay = run_layer(args, rank, world, stream, hbm_peak)

    clk = clocks.stop()

    # ---------------- end to end: host buffers through the C ABI.  Every step uploads its
    # inputs from pinned host memory and downloads its output and final state.  The copies run
    # on their own streams so that PCIe works in both directions at once: the upload of step
    # i + 1 overlaps the prefill and the download of step i (inputs and outputs double-buffered
    # on the device).
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        hg = g.cpu().pin_memory()
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hs = [torch.empty(s_out.shape, dtype=s_out.dtype).pin_memory() for _ in range(2)]
        din = [[torch.empty_like(x) for x in (q, k, v, g)] for _ in range(2)]
        dout = [(torch.empty_like(o), torch.empty_like(s_out)) for _ in range(2)]
        s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            bsel = i & 1
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_done[bsel])   # the prefill that read these buffers is done
                for dst, src in zip(din[bsel], (hq, hk, hv, hg)):
                    dst.copy_(src, non_blocking=True)
                ev_in[bsel].record(s_up)
            stream.wait_event(ev_in[bsel])
            if i >= 2:
                stream.wait_event(ev_out[bsel])      # its output buffers have been downloaded
            dq_, dk_, dv_, dg_ = din[bsel]
            G.gret_prefill_chunkwise(dq_, dk_, dv_, dg_, state_out=dout[bsel][1], o=dout[bsel][0],
                                     workspace=ws)
            ev_done[bsel].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_done[bsel])
                ho[bsel].copy_(dout[bsel][0], non_blocking=True)
                hs[bsel].copy_(dout[bsel][1], non_blocking=True)
                ev_out[bsel].record(s_down)

        for i in range(max(2, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_up.wait_event(e0)
        for i in range(args.steps):
            e2e_step(i)
        stream.wait_stream(s_down)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        if G.gret_workspace_status(ws) != 0:
            raise RuntimeError("prefill reported a timed-out wait in the end-to-end leg")
        bi = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg))
        bo = ho[0].numel() * ho[0].element_size() + hs[0].numel() * hs[0].element_size()
        e2e = {"value": B * N * world * args.steps / (ems * 1e-3) / 1e6, "unit": "Mtok/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
               "ms_per_step": ems / args.steps,
               "overlap": "uploads, prefill and downloads on three streams; step i+1's upload "
                          "overlaps step i's prefill and download"}

    # ---------------- CPU oracle baseline (rank 0 only)
    cpu = None
    if rank == 0 and not args.no_cpu:
        cpu = cpu_baseline(q, k, v, g, args.cpu_tokens)

    line = {
        "metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(world),
        "chunk_sweep": sweep,
        "decode": dec, "varlen_epilogue": epi, "layer": lay,
        "elementwise_gate": ew, "sliding_window": swa, "long_context": long_ctx,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "traffic": prefill_traffic_from_profile(),
                     "kernel": "prefill_tc_kernel", "launch_ms": launch_ms,
                     "algorithmic_bytes_per_launch": alg_bytes},
        "e2e": e2e, "clocks": clk, "gpu_launches": args.steps, "cpu_baseline": cpu,
        # last, so that a record which keeps only the end of the line still has every leg
        "legs": legs_summary(dec, epi, lay, ew, swa, long_ctx),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def legs_summary(dec, epi, lay, ew, swa, long_ctx=None):
    """value, unit and roofline fraction of every secondary leg, rounded, in a few hundred
    characters."""
    def r(x, n=4):
        return None if x is None else float("%.*g" % (n, x))
    out = {}
    if dec:
        out["decode"] = {"v": r(dec["value"]), "u": dec["unit"], "ms": r(dec["ms_per_step"]),
                         "hbm_frac": r(dec["roofline"]["frac"], 3)}
    if epi:
        out["varlen_epilogue"] = {"v": r(epi["value"]), "u": epi["unit"],
                                  "prefill_hbm_frac": r(epi["prefill_roofline"]["frac"], 3),
                                  "gemm_tensor_frac": r(epi["roofline"]["frac"], 3)}
    if lay:
        out["layer"] = {"v": r(lay["value"]), "u": lay["unit"],
                        "proj_tensor_frac": r(lay["roofline"]["frac"], 3),
                        "prefill_hbm_frac": r(lay["prefill_roofline"]["frac"], 3),
                        "gate_tensor_frac": r(lay["gate_roofline"]["frac"], 3)}
    if swa:
        out["sliding_window"] = {"v": r(swa["value"]), "u": swa["unit"],
                                 "tensor_frac": r(swa["roofline"]["frac"], 3)}
        if swa.get("decode"):
            out["sliding_window"]["decode_hbm_frac"] = r(swa["decode"]["roofline"]["frac"], 3)
    if long_ctx:
        out["long_context"] = {"v": r(long_ctx["value"]), "u": long_ctx["unit"],
                               "ms": r(long_ctx["ms_per_step"]),
                               "hbm_frac": r(long_ctx["roofline"]["frac"], 3)}
    if ew:
        out["elementwise_gate"] = {"v": r(ew["value"]), "u": ew["unit"],
                                   "frac": r(ew["roofline"]["frac"], 3),
                                   "bound": ew["roofline"]["bound"],
                                   "x_headwise": r(ew["slowdown_vs_headwise"], 3)}
    return out


def run_long_context(args, rank, world, stream, hbm_peak, peak_kind):
    """The long-context configuration: one sequence of 524288 tokens (4096 chunks), 24 heads of
    128, bf16 q, k, v ~ N(0, 1)/sqrt(128), g ~ N(2, 1), tau 16, the fp32 state carried through
    every chunk; the same kernel and roofline as the headline prefill."""
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI
    Nl = 524288
    inp = SI.gret_inputs(1, Nl, H, D, dtype=torch.bfloat16, g_mean=2.0, g_std=1.0,
                         seed=rank_seed(3, rank), device="cuda")
    q, k, v, g = inp["q"], inp["k"], inp["v"], inp["g"]
    del inp
    o = torch.empty_like(q)
    s_out = torch.empty((1, H, D, D), dtype=torch.float32, device="cuda")
    ws = torch.empty(G.gret_prefill_workspace_size(torch.bfloat16, Nl, 1, H, D, D, 0),
                     dtype=torch.uint8, device="cuda")

    def step():
        G.gret_prefill_chunkwise(q, k, v, g, state_out=s_out, o=o, workspace=ws)

    for _ in range(max(2, min(args.warmup, 3))):
        step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 5))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, world)
    if G.gret_workspace_status(ws) != 0:
        raise RuntimeError("long-context prefill reported a timed-out wait")
    alg = float(Nl * H * BYTES_PER_TOKEN_HEAD)
    ach = alg / (ms * 1e-3) / 1e9
    del q, k, v, g, o, ws
    return {"value": Nl * world / (ms * 1e-3) / 1e6, "unit": "Mtok/s", "tokens": Nl, "heads": H,
            "ms_per_step": ms, "steps": n, "gpu_launches_per_step": 1,
            "l2": "inputs and outputs (12.9 GB) far larger than L2; not flushed",
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                         "frac": ach / hbm_peak, "peak_kind": peak_kind, "traffic": None,
                         "kernel": "prefill_tc_kernel", "algorithmic_bytes_per_launch": alg}}


def run_varlen_epilogue(args, rank, world, stream, hbm_peak):
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI
    lens = SI.varlen_lengths(8, 1024, args.varlen_max_len, seed=5)
    cu = SI.cu_seqlens_of(lens)
    T, Dm = cu[-1], 3072
    inp = SI.gret_inputs(1, T, H, D, dtype=torch.bfloat16, g_mean=0.0, g_std=2.0,
                         seed=rank_seed(5, rank), device="cuda")
    q, k, v, g = (inp[x][0] for x in ("q", "k", "v", "g"))
    del inp
    ep = SI.epilogue_inputs(T, Dm, H * D, seed=rank_seed(5, rank), device="cuda")
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, H * D), dtype=torch.bfloat16, device="cuda")
    need = G.gret_prefill_workspace_size(torch.bfloat16, T, len(lens), H, D, D, 0)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    def step(ev=None):
        G.gret_prefill_chunkwise(q, k, v, g, cu_seqlens=cu_d, o=o, workspace=ws)
        if ev is not None:
            ev.record(stream)
        G.gret_groupnorm_gate(o.view(T, H * D), ep["x"], ep["w_g"], H, y=y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 5))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    barrier(world)
    for i in range(n):
        evs[i][0].record(stream)
        step(evs[i][1])
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    tot_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    epi_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    tot_ms = max_over_ranks(tot_ms, world)
    if G.gret_workspace_status(ws) != 0:
        raise RuntimeError("varlen prefill reported a timed-out wait")
    flops = 2.0 * T * Dm * H * D
    tpeak, tkind = measured_tensor_peak()
    ach = flops / (epi_ms * 1e-3) / 1e12
    pre_bytes = T * H * BYTES_PER_TOKEN_HEAD
    return {"value": T * world / (tot_ms * 1e-3) / 1e6, "unit": "Mtok/s", "tokens": T,
            "lengths": lens, "ms_per_step": tot_ms, "prefill_ms": pre_ms, "epilogue_ms": epi_ms,
            "steps": n, "gpu_launches_per_step": 3,
            "prefill_roofline": {"bound": "hbm", "achieved": pre_bytes / (pre_ms * 1e-3) / 1e9,
                                 "peak": hbm_peak, "unit": "GB/s",
                                 "frac": pre_bytes / (pre_ms * 1e-3) / 1e9 / hbm_peak},
            "roofline": {"bound": "tensor", "achieved": ach, "peak": tpeak, "unit": "TFLOP/s",
                         "frac": ach / tpeak, "peak_kind": tkind + " burst",
                         "traffic": traffic_from_profile("gn_gate.cu",
                                                         "gn_gate_kernel_varlen_T37806.txt", T),
                         "kernel": "gn_gate_kernel", "algorithmic_flops_per_launch": flops}}


# Algorithmic bytes per token and head of the per-channel-gate prefill: q, k, v, o in bf16 and
# one fp32 gate logit per key channel.
EW_BYTES_PER_TOKEN_HEAD = 4 * D * 2 + 4 * D


def run_elementwise(args, rank, world, stream, headwise_ms):
    """The per-key-channel-gate prefill (three launches: range aggregates on the tensor cores,
    scan over ranges, range outputs on the tensor cores) on the 3B shapes, 32768 tokens x 24
    heads, bf16 q, k, v and one fp32 gate logit per key channel.  Also reports the head-wise
    kernel's time on the same shapes over this variant's: the cost of a gate per channel."""
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI
    c = SI.ELEMENTWISE_32K
    Bq, Nq, Hq = c["B"], c["N"], c["H"]
    if args.elementwise_tokens:
        Nq = args.elementwise_tokens
    inp = SI.gret_inputs(Bq, Nq, Hq, D, dtype=torch.bfloat16, seed=rank_seed(c["seed"], rank),
                         device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    del inp
    g = SI.channel_gates(Bq, Nq, Hq, D, g_mean=c["g_mean"], g_std=c["g_std"],
                         seed=rank_seed(c["seed"], rank), device="cuda")
    o = torch.empty_like(q)
    s_out = torch.empty((Bq, Hq, D, D), dtype=torch.float32, device="cuda")
    ws = torch.empty(G.gret_prefill_elementwise_workspace_size(Bq, Nq, Hq, D),
                     dtype=torch.uint8, device="cuda")

    def step():
        G.gret_prefill_elementwise(q, k, v, g, state_out=s_out, o=o, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, world)
    if G.gret_workspace_status(ws) != 0:
        raise RuntimeError("per-channel prefill reported a timed-out wait")
    tokens = Bq * Nq
    alg = float(EW_BYTES_PER_TOKEN_HEAD) * tokens * Hq
    ach = alg / (ms * 1e-3) / 1e9
    peak, kind = measured_peaks()
    return {"value": tokens * world / (ms * 1e-3) / 1e6, "unit": "Mtok/s", "tokens": tokens,
            "heads": Hq, "ms_per_step": ms, "steps": n, "gpu_launches_per_step": 3,
            "gate": "one logit per key channel, g ~ N(2, 1)",
            "headwise_ms_same_shapes": headwise_ms,
            "slowdown_vs_headwise": ms / headwise_ms,
            "workspace_bytes": ws.numel(),
            "l2": "inputs and outputs (1.2 GB) larger than L2; not flushed",
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": ach / peak, "peak_kind": kind,
                         "traffic": traffic_from_profile("prefill_ew.cu",
                                                         "ew_kernels_32k.txt", Nq),
                         "kernel": "ew_range_state + ew_state_scan + ew_range_output",
                         "algorithmic_bytes_per_launch": alg}}


def run_swa(args, rank, world, stream, headwise_ms):
    """Sliding-window softmax attention (window 1024) on the 3B shapes, 32768 tokens x 24 heads
    of 128, bf16: one launch per step.  FLOP counted algorithmically, 4 d per (query, visible
    key) pair (Q K^T and P V)."""
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI
    c = SI.SWA_32K
    Bq, Nq, Hq, W = c["B"], c["N"], c["H"], c["window"]
    inp = SI.gret_inputs(Bq, Nq, Hq, D, dtype=torch.bfloat16, seed=rank_seed(c["seed"], rank),
                         device="cuda")
    q = (inp["q"] * D ** 0.5).to(torch.bfloat16)
    k = (inp["k"] * D ** 0.5).to(torch.bfloat16)
    v = inp["v"]
    del inp
    o = torch.empty_like(q)

    def step():
        G.gret_swa_prefill(q, k, v, window=W, o=o)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, world)
    del q, k, v, o
    dec = run_swa_decode(args, rank, world, stream, W)
    pairs = W * (W + 1) // 2 + (Nq - W) * W if Nq >= W else Nq * (Nq + 1) // 2
    flops = 4.0 * D * pairs * Hq * Bq
    tpeak, tkind = measured_tensor_peak()
    ach = flops / (ms * 1e-3) / 1e12
    return {"value": Bq * Nq * world / (ms * 1e-3) / 1e6, "unit": "Mtok/s", "tokens": Bq * Nq,
            "heads": Hq, "window": W, "ms_per_step": ms, "steps": n, "gpu_launches_per_step": 1,
            "gated_retention_ms_same_shapes": headwise_ms,
            "l2": "q, k, v, o (805 MB) larger than L2; not flushed",
            "roofline": {"bound": "tensor", "achieved": ach, "peak": tpeak, "unit": "TFLOP/s",
                         "frac": ach / tpeak, "peak_kind": tkind + " burst",
                         "mma": "tcgen05 bf16, S and O in TMEM",
                         "traffic": traffic_from_profile("swa_tc.cu",
                                                         "swa_tc_kernel_32k_w1024.txt"),
                         "kernel": "swa_tc_kernel", "algorithmic_flops_per_launch": flops},
            "decode": dec}


SWA_DEC_B, SWA_DEC_STEPS = 64, 64


def run_swa_decode(args, rank, world, stream, W):
    """Sliding-window decode with a full ring-buffer cache: 64 sequences x 24 heads of 128,
    window W, each step one token per sequence (positions 4096 .. 4096 + steps - 1, so every
    step reads a whole window).  HBM-bound: per (b, h) and step the window's keys and values
    (2 W d 2 bytes), q, k, v, o and the cache slot written."""
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI
    hbm_peak, peak_kind = measured_peaks()
    Bq, Hq, S = SWA_DEC_B, H, SWA_DEC_STEPS
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(9, rank))
    kc = torch.randn((Bq, Hq, W, D), generator=gen, device="cuda").to(torch.bfloat16)
    vc = (torch.randn((Bq, Hq, W, D), generator=gen, device="cuda") * D ** -0.5).to(torch.bfloat16)
    st = SI.gret_inputs(Bq, S, Hq, D, dtype=torch.bfloat16, seed=rank_seed(90, rank),
                        device="cuda")
    qs = (st["q"] * D ** 0.5).to(torch.bfloat16).permute(1, 0, 2, 3).contiguous()
    ks = (st["k"] * D ** 0.5).to(torch.bfloat16).permute(1, 0, 2, 3).contiguous()
    vs = st["v"].permute(1, 0, 2, 3).contiguous()
    del st
    pos = [torch.full((Bq,), 4096 + i, dtype=torch.int32, device="cuda") for i in range(S)]
    od = torch.empty((Bq, Hq, D), dtype=torch.bfloat16, device="cuda")
    for i in range(args.warmup):
        G.gret_swa_decode_step(qs[i], ks[i], vs[i], pos[i], kc, vc, o=od)
    torch.cuda.synchronize()
    barrier(world)
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for i in range(S):
        G.gret_swa_decode_step(qs[i], ks[i], vs[i], pos[i], kc, vc, o=od)
    d1.record(stream)
    torch.cuda.synchronize()
    dms = max_over_ranks(d0.elapsed_time(d1), world)
    per_bh = 2 * W * D * 2 + 4 * D * 2 + 2 * D * 2
    ach = Bq * Hq * per_bh / (dms / S * 1e-3) / 1e9
    return {"value": Bq * S * world / (dms * 1e-3), "unit": "tok/s", "ms_per_step": dms / S,
            "batch": Bq, "window": W, "steps": S, "gpu_launches": S,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                         "frac": ach / hbm_peak, "peak_kind": peak_kind,
                         "traffic": traffic_from_profile("swa_decode.cu",
                                                         "swa_decode_kernel_bs64_w1024.txt"),
                         "kernel": "swa_decode_kernel",
                         "algorithmic_bytes_per_launch": Bq * Hq * per_bh}}


def run_layer(args, rank, world, stream, hbm_peak):
    """One gated-retention mixer layer at the 3B shapes (32768 tokens of one sequence, hidden
    3072, 24 heads of 128): the [q | k | v | g] = x W projection (one tcgen05 GEMM), the
    chunkwise prefill (k scaled by d^-1/2) and the GroupNorm * swish(x W_G) output gate, with
    events between the three launches on the launching stream."""
    import torch

    import gated_retention_linear_b200 as G
    import synth_inputs as SI
    c = SI.LAYER_32K
    T, Dm, Hh, d = c["T"], c["D"], c["H"], c["dk"]
    F = 3 * Hh * d + Hh
    li = SI.layer_inputs(T, Dm, Hh, d, seed=rank_seed(c["seed"], rank), device="cuda",
                         pad=(-F) % 8, pad_value=0.0)
    x, w, w_g = li["x"], li["w_qkvg"], li["w_g"]
    cu_d = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    o = torch.empty((T, Hh, d), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, Hh * d), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(G.gret_prefill_workspace_size(torch.bfloat16, T, 1, Hh, d, d, 0),
                     dtype=torch.uint8, device="cuda")

    def step(ev=None):
        q, k, v, g = G.gret_qkvg_projection(x, w, Hh, d)
        if ev is not None:
            ev[1].record(stream)
        G.gret_prefill_chunkwise(q, k, v, g, k_scale=d ** -0.5, cu_seqlens=cu_d, o=o,
                                 workspace=ws)
        if ev is not None:
            ev[2].record(stream)
        G.gret_groupnorm_gate(o.view(T, Hh * d), x, w_g, Hh, y=y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 5))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    barrier(world)
    for i in range(n):
        evs[i][0].record(stream)
        step(evs[i])
        evs[i][3].record(stream)
    torch.cuda.synchronize()
    tot_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[3]) for e in evs), world)
    proj_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    pre_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    gn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    if G.gret_workspace_status(ws) != 0:
        raise RuntimeError("layer prefill reported a timed-out wait")
    tpeak, tkind = measured_tensor_peak()
    proj_flops = 2.0 * T * Dm * F
    gn_flops = 2.0 * T * Dm * Hh * d
    pre_bytes = T * Hh * BYTES_PER_TOKEN_HEAD
    ach = proj_flops / (proj_ms * 1e-3) / 1e12
    return {"value": T * world / (tot_ms * 1e-3) / 1e6, "unit": "Mtok/s", "tokens": T,
            "hidden": Dm, "heads": Hh, "ms_per_step": tot_ms, "projection_ms": proj_ms,
            "prefill_ms": pre_ms, "gate_ms": gn_ms, "steps": n, "gpu_launches_per_step": 4,
            "l2": "x (201 MB) and q, k, v (604 MB) larger than L2 (126 MB); not flushed",
            "roofline": {"bound": "tensor", "achieved": ach, "peak": tpeak, "unit": "TFLOP/s",
                         "frac": ach / tpeak, "peak_kind": tkind + " burst", "traffic": None,
                         "kernel": "qkvg_projection (gn_gate_kernel<EPI_PROJECTION>)",
                         "algorithmic_flops_per_launch": proj_flops},
            "prefill_roofline": {"bound": "hbm", "achieved": pre_bytes / (pre_ms * 1e-3) / 1e9,
                                 "peak": hbm_peak, "unit": "GB/s",
                                 "frac": pre_bytes / (pre_ms * 1e-3) / 1e9 / hbm_peak},
            "gate_roofline": {"bound": "tensor",
                              "achieved": gn_flops / (gn_ms * 1e-3) / 1e12, "peak": tpeak,
                              "unit": "TFLOP/s",
                              "frac": gn_flops / (gn_ms * 1e-3) / 1e12 / tpeak}}


def cpu_baseline(q, k, v, g, n_tokens, min_seconds=8.0, max_reps=8):
    """The fp64 oracle, as it stands, on the first n_tokens tokens of all 24 heads, repeated until
    about min_seconds of CPU work have been timed (at most max_reps passes)."""
    from oracle import oracle
    n = min(n_tokens, N)
    qc = q[0, :n].cpu()
    kc = k[0, :n].cpu()
    vc = v[0, :n].cpu()
    gc = g[0, :n].cpu()
    reps, dt = 0, 0.0
    while reps < max_reps and (reps == 0 or dt < min_seconds):
        t0 = time.perf_counter()
        oracle.gret_recurrent(qc, kc, vc, gc)
        dt += time.perf_counter() - t0
        reps += 1
    return {"value": n * reps / dt / 1e6, "unit": "Mtok/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": "%d tokens x 24 heads, fp64 recurrent oracle, %d passes, %.1f s"
                      % (n, reps, dt)}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on host cores (rank 0 only under torchrun)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    import synth_inputs as SI
    from oracle import oracle
    n = min(args.cpu_tokens, N)
    inp = SI.gret_inputs(1, n, H, D, dtype=torch.bfloat16, seed=2, device="cpu")
    q, k, v, g = (inp[x][0] for x in ("q", "k", "v", "g"))
    for _ in range(args.warmup):
        oracle.gret_recurrent(q, k, v, g)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gret_recurrent(q, k, v, g)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt / 1e6
    sample = ("first %d of 32768 tokens of the 3B-shaped prefill, all 24 heads, fp64 recurrent "
              "oracle per step" % n)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=32768)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-epilogue", action="store_true")
    ap.add_argument("--no-layer", action="store_true")
    ap.add_argument("--no-elementwise", action="store_true")
    ap.add_argument("--no-swa", action="store_true")
    ap.add_argument("--no-long", action="store_true",
                    help="skip the long-context leg (524288 tokens x 24 heads, 13 GB)")
    ap.add_argument("--elementwise-tokens", type=int, default=None,
                    help="tokens of the per-channel-gate leg (default: the 32768 of its "
                         "workload; smaller values are for profiling captures)")
    ap.add_argument("--chunk-sweep", action="store_true",
                    help="also time the 3B-shaped prefill at every chunk size the library takes "
                         "(16, 32, 64 on CUDA cores, 128 on the tensor cores)")
    ap.add_argument("--varlen-max-len", type=int, default=65536,
                    help="longest sequence of the varlen + epilogue leg (a smaller value gives "
                         "a small case for profiling)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    if args.impl == "reference":
        if args.cpu_tokens == 32768:
            args.cpu_tokens = 4096
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
