"""Benchmark of the mask-free spatially adaptive DiT attention path on B200.

One step = one denoising trajectory of the 2560^2-equivalent workload
(B=2 cond/uncond, H=24, N=25600 image tokens, d=96, L=256 text tokens with 128
valid, |S| = 0.3 N = 7680): 10 denoising steps with dense anchors at t = 0, 5;
t = 0 is also the PCSP warm-up (cross-attention probabilities -> score), the
S/C split follows it, the image mask is checked once, every SRSU step
scatters the fresh S-row K/V into the cached state and runs subset attention
with the output scattered into O_state, and every step ends with the
guidance combine.  Every row of the hot path runs in libsafedit.so kernels.

value = SRSU subset-attention TFLOP/s (4 k N d B H flop per call) over all SRSU
launches of the timed steps, timed with CUDA events on the launching stream;
whole-job aggregate over ranks (sum of flop / max of per-rank time).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
(for N > 1 launch under torchrun; by default each rank runs its own independent
replica; --shard heads splits one generation by heads, --shard cfg on 2 GPUs by
guidance branch).
"""
import argparse
import json
import re
import os
import statistics
import subprocess
import tempfile
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from spatially_adaptive_dit_b200 import workloads as wl  # noqa: E402

METRIC = "SRSU subset-attention TFLOP/s & ms at N=25600,|S|=0.3N; partition/CFG HBM GB/s"
W = wl.W2560
WORKLOAD = ("2560^2-equivalent: B=2 (cond/uncond), H=24, N=25600 (160x160), d=96, L=256 (128 valid), "
            "|S|=0.3N=7680, 10-step trajectory with anchors at t=0,5 (t=0 = PCSP warm-up)")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def percentiles(ms):
    """p10 / p50 / p90 (nearest rank) of a list of timings."""
    v = sorted(ms)
    pick = lambda q: v[int(round(q * (len(v) - 1)))]
    return {"p10": round(pick(0.1), 4), "p50": round(pick(0.5), 4), "p90": round(pick(0.9), 4)}


class L2Flush:
    """Writes a buffer of four times the L2 size, so that the next launch finds
    none of its inputs in L2, then reads it back, so that the lines left in L2
    are clean and the timed launch does not pay for writing them back (run
    between timed repetitions, outside the events)."""

    def __init__(self, dev):
        self.bytes = 4 * torch.cuda.get_device_properties(dev).L2_cache_size
        self.buf = torch.empty(self.bytes // 4, dtype=torch.int32, device=dev)
        self.sink = torch.empty((), dtype=torch.int32, device=dev)

    def __call__(self):
        self.buf.fill_(1)
        torch.amax(self.buf, dim=0, out=self.sink)


def time_reps_interleaved(fns, stream, reps=20, warmup=3):
    """Like time_reps for several launches at once, taken in turn within every
    repetition (so that clock and power drift over the run affects them
    alike).  Returns name -> p10 / p50 / p90."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            for fn in fns.values():
                fn()
        evs = {n: [] for n in fns}
        for _ in range(reps):
            for n, fn in fns.items():
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                evs[n].append((a, b))
    stream.synchronize()
    out = {}
    for n, lst in evs.items():
        out[n] = percentiles([a.elapsed_time(b) for a, b in lst])
        out[n]["n"] = reps
    return out


def time_reps(fn, stream, reps=20, warmup=3, flush=None):
    """CUDA-event timings (ms) of `reps` launches of fn() on `stream` after
    `warmup` untimed ones; `flush` (optional) runs before every launch,
    outside the events.  Returns p10 / p50 / p90 and the sample count."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
        evs = []
        for _ in range(reps):
            if flush is not None:
                flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            evs.append((a, b))
    stream.synchronize()
    out = percentiles([a.elapsed_time(b) for a, b in evs])
    out["n"] = reps
    return out


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        try:
            self.dev = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.dev = str(device_index)
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"safedit_clocks_dev{device_index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
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
        for ln in open(self.path):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        busy = [x for x in sm if x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def head_range(H, world, rank):
    """Heads [h0, h1) of rank `rank` when one generation's H heads are split
    evenly over `world` GPUs."""
    if H % world != 0:
        raise ValueError(f"{H} heads do not split evenly over {world} GPUs")
    n = H // world
    return rank * n, (rank + 1) * n


def score_all_reduce(score):
    """The one exchange of a head-sharded generation: the fp64 PCSP score
    vector (each rank's sum over its own heads) summed over all ranks, so
    that every rank makes the identical S/C split."""
    torch.distributed.all_reduce(score, op=torch.distributed.ReduceOp.SUM)


def split_broadcast(tr):
    """CFG-parallel generation: the S/C split and the sensitivity score are
    made on the cond-branch rank (0), which alone has a prompt to score
    against, and sent to the uncond-branch rank."""
    for t in (tr.idx_s, tr.idx_c, tr.s):
        torch.distributed.broadcast(t, src=0)


def eps_all_gather(tr):
    """CFG-parallel generation: each rank's branch prediction (rank 0 the
    conditional, rank 1 the unconditional one) to both ranks, before the
    guidance combine that needs the two."""
    torch.distributed.all_gather([tr.eps_c, tr.eps_u], tr.eps_own)


class Trajectory:
    """Device-resident buffers and the launch sequence of one trajectory.
    heads=(h0, h1) keeps only those heads of the (same, globally seeded)
    generation on this device; reduce_score then completes the PCSP score
    over the other devices' heads before the split.  branch=b keeps only
    batch entry b (0 = cond, 1 = uncond) of the self-attention tensors and of
    the prediction; only the cond branch scores the tokens, share_split then
    hands the split to the other branch's device, and exchange_eps gathers
    both branches' predictions before every guidance combine."""

    def __init__(self, w, dev, seed_step=0, heads=None, reduce_score=None, pcsp="fused", branch=None,
                 share_split=None, exchange_eps=None):
        from spatially_adaptive_dit_b200 import safedit as sd
        self.sd, self.w, self.dev = sd, w, dev
        self.pcsp = pcsp  # "fused": one pcsp_score launch; "unfused": probabilities, then aggregation
        N, d, L, k = w.N, w.d, w.L, w.k
        h0, h1 = (0, w.H) if heads is None else heads
        b0, b1 = (0, w.B) if branch is None else (branch, branch + 1)
        H, B = h1 - h0, b1 - b0
        slh = (lambda t: t) if heads is None else (lambda t: t[:, h0:h1].contiguous())
        sl = (lambda t: slh(t)) if branch is None else (lambda t: slh(t)[b0:b1].contiguous())
        self.reduce_score = reduce_score
        self.branch, self.share_split, self.exchange_eps = branch, share_split, exchange_eps
        self.pcsp_here = branch in (None, 0)  # the score comes from the cond branch
        self.k = k
        self.q, self.k_full, self.v_full = (sl(t) for t in wl.qkv(w, step=seed_step, device=dev))
        self.k_s, self.v_s = (sl(t) for t in wl.fresh_sensitive_kv(w, k, step=seed_step, device=dev))
        self.k_state = torch.empty_like(self.k_full)
        self.v_state = torch.empty_like(self.v_full)
        self.k_state.copy_(self.k_full)
        self.v_state.copy_(self.v_full)
        self.o_state = torch.zeros_like(self.q)
        self.q_img, self.k_txt, self.valid, self.content = wl.text(w, step=seed_step, device=dev)
        self.q_img, self.k_txt = slh(self.q_img), slh(self.k_txt)
        self.P = torch.empty(H, N, L, device=dev)
        self.score = torch.zeros(N, dtype=torch.float64, device=dev)
        self.idx_s = torch.empty(k, dtype=torch.int32, device=dev)
        self.idx_c = torch.empty(N - k, dtype=torch.int32, device=dev)
        self.s = torch.zeros(N, device=dev)
        # Image self-attention mask as the backbone passes it: an all-valid key
        # mask broadcast over queries ([B,1,1,N] -> [B,1,N,N]).
        self.mask = torch.zeros(B, 1, 1, N, dtype=torch.bfloat16, device=dev).expand(B, 1, N, N)
        self.verdict = torch.zeros(1, dtype=torch.int32, device=dev)
        self.eps_c, self.eps_u = wl.cfg_preds(w, step=seed_step, device=dev)
        self.eps_own = None if branch is None else (self.eps_c, self.eps_u)[branch].clone()
        self.cfg_out = torch.empty_like(self.eps_c)
        self.H, self.B = H, B
        # tail-balanced attention: one workspace per launch shape (S rows,
        # all rows), as large as the launch plan asks (none where it keeps
        # whole units, as at 2560^2)
        self.attn_ws = {}
        for rows in (k, N):
            nb = sd.safedit_attn_subset_workspace_size(B, H, rows, N, d)
            self.attn_ws[rows] = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
        self.flop_srsu = 4.0 * k * N * d * B * H
        self.flop_dense = 4.0 * N * N * d * B * H
        self.bytes = {
            "cross_attn_probs": H * N * L * 4 + H * N * d * 2 + H * L * d * 2,
            # Q_img and K_txt of the cond branch read once, the fp64 score read and written
            "pcsp_score": H * N * d * 2 + H * L * d * 2 + 2 * N * 8,
            # the 16-byte groups of P that hold a content column (the kernel reads no others)
            "partition_accumulate": H * N * 16 * int(self.content.view(-1, 4).any(dim=1).sum()) + N * 16 + L,
            "scatter_state": 2 * (2 * B * H * k * d * 2) + 4 * k,
            "sw_cfg": 3 * N * w.F * 4 + 4 * N,
        }

    def attn(self, q, k_state, v_state, idx, n_idx, out, scattered, stream):
        """One attention launch through the tail-balanced entry point."""
        rows = n_idx if idx is not None else q.shape[2]
        self.sd.safedit_attn_subset_ws(q, k_state, v_state, idx, n_idx, None, None, 0.0, out, scattered,
                                       self.attn_ws[rows], stream)

    def run(self, stream, ev=None, flush=None):
        """Enqueue one trajectory on `stream`.  ev: dict name -> list to which
        (start, end) CUDA events of each launch are appended.  flush: called
        before every attention and scatter launch, outside its events (an L2
        flush where the per-device state would otherwise stay in L2)."""
        sd, w = self.sd, self.w

        def timed(name, fn):
            if flush is not None and name in ("attn_dense_anchor", "attn_subset_srsu", "scatter_state"):
                flush()
            if ev is None:
                fn()
                return
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ev.setdefault(name, []).append((a, b))

        self.score.zero_()
        for t in range(w.steps):
            anchor = (t % w.period == 0)
            if t < w.warmup and self.pcsp_here and self.pcsp == "fused":  # PCSP warm-up on the cond branch
                timed("pcsp_score", lambda: sd.safedit_pcsp_score(
                    self.q_img, self.k_txt, self.valid, self.content, 0, 0.0, self.score, stream))
            elif t < w.warmup and self.pcsp_here:
                timed("cross_attn_probs", lambda: sd.safedit_cross_attn_probs(
                    self.q_img, self.k_txt, self.valid, 0, 0.0, self.P, stream))
                timed("partition_accumulate", lambda: sd.safedit_partition_accumulate(
                    self.P, self.content, self.score, stream))
            if t == w.warmup - 1 and self.reduce_score is not None:
                timed("score_all_reduce", lambda: self.reduce_score(self.score))
            if t == w.warmup - 1 and self.pcsp_here:
                timed("partition_finalize", lambda: sd.safedit_partition_finalize(
                    self.score, w.N, self.k, self.idx_s, self.idx_c, self.s, stream))
            if t == w.warmup - 1 and self.share_split is not None:
                timed("split_broadcast", lambda: self.share_split(self))
            if t == 0:
                timed("mask_is_row_constant", lambda: sd.safedit_mask_is_row_constant(
                    self.mask, self.verdict, None, stream))
            if anchor:
                # CAR: fresh K/V become the cached state (buffer swap), dense refresh of all rows
                self.k_state, self.k_full = self.k_full, self.k_state
                self.v_state, self.v_full = self.v_full, self.v_state
                timed("attn_dense_anchor", lambda: self.attn(
                    self.q, self.k_state, self.v_state, None, 0, self.o_state, 0, stream))
            else:
                timed("scatter_state", lambda: sd.safedit_scatter_state(
                    [self.k_s, self.v_s], [self.k_state, self.v_state], self.idx_s, self.k, stream))
                timed("attn_subset_srsu", lambda: self.attn(
                    self.q, self.k_state, self.v_state, self.idx_s, self.k, self.o_state, 1, stream))
            g_ctx = w.gamma_ctx
            g_sens = w.gamma_sens if t >= w.warmup else w.gamma_ctx  # global CFG before the split
            if self.exchange_eps is not None:
                timed("eps_exchange", lambda: self.exchange_eps(self))
            timed("sw_cfg", lambda: sd.safedit_sw_cfg(self.eps_c, self.eps_u, self.s, g_ctx, g_sens,
                                                       self.cfg_out, stream))


def run_ours(args):
    ws, rank, local = _dist()
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from spatially_adaptive_dit_b200 import safedit as sd
    sharded = args.shard in ("heads", "cfg") and ws > 1
    if sharded and args.shard == "cfg":
        # one generation, its cond / uncond branches on two GPUs: the split
        # broadcast once, the branch predictions gathered every step
        if ws != 2:
            raise SystemExit("--shard cfg puts the two guidance branches on exactly 2 GPUs")
        tr = Trajectory(W, dev, seed_step=0, branch=rank, share_split=split_broadcast,
                        exchange_eps=eps_all_gather, pcsp=args.pcsp)
    elif sharded:  # one generation, H / ws heads per GPU, one score all-reduce
        tr = Trajectory(W, dev, seed_step=0, heads=head_range(W.H, ws, rank), reduce_score=score_all_reduce,
                        pcsp=args.pcsp)
    else:  # independent replicas
        tr = Trajectory(W, dev, seed_step=1000 * rank, pcsp=args.pcsp)
    torch.cuda.synchronize()
    # the peak below counts the trajectory's own buffers, not the temporaries of their construction
    torch.cuda.reset_peak_memory_stats(dev)
    # L2: this device's K/V state must not be served from L2 between launches
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    state_bytes = tr.k_state.numel() * tr.k_state.element_size()
    flush = L2Flush(dev) if 2 * state_bytes < 2 * l2 else None
    l2_note = (f"per-device K/V state {2 * state_bytes / 1e6:.0f} MB under twice the L2 ({l2 / 1e6:.0f} MB): L2 flushed "
               f"({4 * l2 / 1e6:.0f} MB write) before every attention and scatter launch, outside their events"
               if flush is not None else
               f"inputs larger than L2 (Q/K/V/state {state_bytes / 1e6:.0f} MB each per device, L2 "
               f"{l2 / 1e6:.0f} MB), no flush needed")
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            tr.run(stream, flush=flush)
    stream.synchronize()
    assert sd.safedit_get_device_status(stream) == 0

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = {}
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = sd.safedit_kernel_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            tr.run(stream, ev, flush=flush)
    t1.record(stream)
    t1.synchronize()
    torch.cuda.synchronize()
    launches = sd.safedit_kernel_launch_count() - n0
    if ws > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    status = sd.safedit_get_device_status(stream)
    peak_gb = torch.cuda.max_memory_allocated(dev) / 1e9
    total_ms = t0.elapsed_time(t1)
    per = {n: [a.elapsed_time(b) for a, b in lst] for n, lst in ev.items()}
    srsu_ms = sum(per["attn_subset_srsu"])
    n_srsu = len(per["attn_subset_srsu"])
    total_ms, srsu_ms = max_over_ranks([total_ms, srsu_ms], dev)

    # ---- end to end through the public API with host buffers (pinned)
    e2e = run_e2e(tr, stream, args)
    e2e["ms"] = max_over_ranks([e2e["ms"]], dev)[0]
    # the unfused PCSP rows (probabilities, then aggregation), each launched alone
    rows_flush = L2Flush(dev)
    alone = {
        "cross_attn_probs": time_reps(lambda: sd.safedit_cross_attn_probs(
            tr.q_img, tr.k_txt, tr.valid, 0, 0.0, tr.P, stream), stream, flush=rows_flush),
        "partition_accumulate": time_reps(lambda: sd.safedit_partition_accumulate(
            tr.P, tr.content, tr.score, stream), stream, flush=rows_flush),
    }
    del rows_flush
    unfused = alone["cross_attn_probs"]["p50"] + alone["partition_accumulate"]["p50"]
    ext = measure_extensions(tr, stream, dev, unfused)

    if rank == 0:
        hbm, bf16_burst, bf16_sust, src = _peaks()
        value = whole_job_tflops(tr.flop_srsu * n_srsu, ws, srsu_ms)
        srsu_call_ms = srsu_ms / n_srsu
        achieved = tr.flop_srsu / (srsu_call_ms * 1e-3) / 1e12
        kern = {}

        def bw(entry, name, ms):
            if name in tr.bytes:
                gbs = tr.bytes[name] / (ms * 1e-3) / 1e9
                entry.update({"gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)})

        for n, v in per.items():
            m = statistics.mean(v)
            entry = {"ms_mean": round(m, 4), "calls_per_step": len(v) // args.steps, **percentiles(v),
                     "n": len(v), "timed": "inside the trajectory"}
            bw(entry, n, entry["p50"])
            if n == "attn_dense_anchor":
                entry["tflops"] = round(tr.flop_dense / (m * 1e-3) / 1e12, 1)
            if n == "attn_subset_srsu":
                entry["tflops"] = round(tr.flop_srsu / (m * 1e-3) / 1e12, 1)
            kern[n] = entry
        for n, t in alone.items():
            entry = {**t, "timed": "launched alone, 3 warm-ups + 20 reps, L2 flushed before each"}
            bw(entry, n, t["p50"])
            kern[n] = entry
        traffic = _ncu_traffic()
        algo_bytes = _srsu_algorithmic_bytes(tr)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 3),
            "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": W.B if sharded else W.B * ws, "seq_len": W.N,
                       "parallelism": ("cfg x2 (one generation, its cond and uncond branches on one GPU each; "
                                       "the S/C split and s broadcast once from the cond branch, the two "
                                       "branch predictions all-gathered before every guidance combine)")
                                      if sharded and args.shard == "cfg" else
                                      (f"heads x{ws} (one generation, {W.H // ws} heads per GPU; one all-reduce "
                                       "of the fp64 score vector after the warm-up)") if sharded else
                                      f"replicas x{ws} (independent trajectories, no collective)",
                       "l2": l2_note,
                       "pcsp": ("fused pcsp_score on the warm-up step" if tr.pcsp == "fused" else
                                "cross_attn_probs + partition_accumulate on the warm-up step"),
                       "srsu_calls_per_step": n_srsu // args.steps,
                       "srsu_ms_per_call": round(srsu_call_ms, 4)},
            "kernels": kern,
            "roofline": {"kernel": "attn_subset (SRSU)", "bound": "tensor", "achieved": round(achieved, 1),
                         "peak": bf16_sust, "peak_kind": f"bf16_tflops_sustained ({src})",
                         "unit": "TFLOP/s", "frac": round(achieved / bf16_sust, 4),
                         "frac_of_burst": round(achieved / bf16_burst, 4),
                         # the same call at the SM clock the burst peak runs at: the power cap's
                         # clock (median under load) against the maximum
                         "frac_of_burst_at_max_clock": (round(achieved * clk["sm_max_mhz"] / clk["sm_mhz"] /
                                                              bf16_burst, 4)
                                                        if clk and clk.get("sm_mhz") else None),
                         "traffic": traffic,
                         "algorithmic_bytes": algo_bytes,
                         "traffic_over_algorithmic": None if traffic is None else round(traffic / algo_bytes, 3),
                         "mufu_colimit": mufu_colimit(W.d, 0.75)},
            "gpu_launches": launches,
            "memory": {"peak_allocated_gb": round(peak_gb, 2),
                       "note": f"this device's buffers of the attention path ({tr.H} heads) incl. the "
                               f"{tr.P.numel() * 4 / 1e9:.2f} GB probability tensor; a dense masked path that "
                               "materialises bf16 scores [B,H,N,N] would need "
                               f"{tr.B * tr.H * W.N * W.N * 2 / 1e9:.1f} GB for them alone"},
            "device_status": status,
            "extensions": ext,
            "e2e": {"value": round(whole_job_tflops(tr.flop_srsu * n_srsu / args.steps, ws, e2e["ms"]), 3),
                    "unit": "TFLOP/s", "ms_per_step": round(e2e["ms"], 3),
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
            "clocks": clk,
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
            gms = {n: e.get("p50", e.get("ms_mean")) for n, e in kern.items()}
            gms.update({"ffn_block": ext["ffn_block"]["p50"], "mask_is_row_constant": ext["mask_stress"]["p50"],
                        "qkv_projection_gathered": ext["qkv_projection_gathered"]["p50"],
                        "stepcache_sw_cfg": ext["stepcache_sw_cfg"]["p50"]})
            line["oracle_rows"] = oracle_rows(gms)
            g1024 = {n: e["p50"] for n, e in ext["config_1024"].items() if isinstance(e, dict) and "p50" in e}
            line["oracle_1024"] = oracle_full_1024(g1024)
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def mufu_colimit(d, mufu_share):
    """Ceiling the exponentials put on the attention, as a fraction of the
    tensor peak: per (query, key) pair the MMAs do 4 d flop at 8192 dense bf16
    flop per clock per SM, and the softmax one exponential, of which
    `mufu_share` runs on the MUFU unit at 16 per clock per SM (measured on
    B200) and the rest on the FMA pipe."""
    tensor_clk, mufu_clk = 4 * d / 8192, mufu_share / 16
    return {"flop_per_exponential": 4 * d, "tensor_flop_per_clk_sm": 8192, "ex2_per_clk_sm": 16,
            "ceiling_all_on_mufu": round(min(1.0, tensor_clk / (1 / 16)), 3),
            "mufu_share_as_built": mufu_share,
            "ceiling_as_built": round(min(1.0, tensor_clk / mufu_clk), 3)}


def _srsu_algorithmic_bytes(tr):
    """Bytes one SRSU launch must move at least: K and V of every slice read
    once, the gathered Q rows read and the output rows written."""
    w = tr.w
    return (2 * w.N + 2 * tr.k) * w.d * 2 * tr.B * tr.H + 4 * tr.k


def measure_extensions(tr, stream, dev, unfused_pcsp_ms):
    """The steps around the per-step path and the other configurations, each
    launched alone (3 warm-ups + 20 CUDA-event reps, p50 with p10 / p90; L2
    flushed before every rep wherever the inputs could stay in L2): the fused
    PCSP score, SkipSparse's projections on the focus rows (gathered Q|K|V;
    FFN W1 with bias and GELU; FFN W2 with bias, rows scattered into the FFN
    cache), the StepCache guidance combine, the mask check and the kept-mask
    SRSU calls of the stress shape, the 1024^2 configuration, the 3072^2
    sensitive-fraction sweep and the guidance combines at F = 4096."""
    sd, w = tr.sd, tr.w
    hbm, bf16_burst, _, src = _peaks()
    k, D, F, B = tr.k, w.D_model, w.D_ff, w.B
    flush = L2Flush(dev)
    w1, b1, w2, b2 = (t.to(dev) for t in wl.ffn_weights(w))
    wqkv, bqkv = (t.to(dev) for t in wl.qkv_proj_weights(w))
    x, y = (t.to(dev) for t in wl.ffn_states(w))
    xs = torch.empty(B, 1, k, D, dtype=torch.bfloat16, device=dev)
    xs3 = xs.view(B, k, D)
    h = torch.empty(B, k, F, dtype=torch.bfloat16, device=dev)
    qkv = torch.empty(B, k, 3 * D, dtype=torch.bfloat16, device=dev)
    prev_c, prev_u = wl.cfg_preds(w, step=1, device=dev)

    def gemm_entry(t, flop):
        tf = flop / (t["p50"] * 1e-3) / 1e12
        return {**t, "tflops": round(tf, 1), "frac": round(tf / bf16_burst, 3),
                "peak": bf16_burst, "peak_kind": f"bf16_tflops burst ({src})"}

    def bw_entry(t, nbytes, note=None):
        gbs = nbytes / (t["p50"] * 1e-3) / 1e9
        e = {**t, "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)}
        if note:
            e["note"] = note
        return e

    gather = lambda: sd.safedit_gather_rows([x.view(B, 1, w.N, D)], [xs], tr.idx_s, k, stream)
    ffn1 = lambda: sd.safedit_gemm_bias_act(xs3, w1, b1, 1, None, h, stream)
    ffn2 = lambda: sd.safedit_gemm_bias_act(h, w2, b2, 0, tr.idx_s, y, stream)
    proj = lambda: sd.safedit_gemm_bias_act(xs3, wqkv, bqkv, 0, None, qkv, stream)
    gather()
    ffn_flop = 2.0 * B * k * D * F
    pcsp = time_reps(lambda: sd.safedit_pcsp_score(tr.q_img, tr.k_txt, tr.valid, tr.content, 0, 0.0, tr.score,
                                                   stream), stream, flush=flush)
    out = {
        "pcsp_fused": {**pcsp, "unfused_ms": round(unfused_pcsp_ms, 4)},
        "qkv_projection_gathered": gemm_entry(time_reps(proj, stream), 2.0 * B * k * D * 3 * D),
        "ffn_w1_bias_gelu": gemm_entry(time_reps(ffn1, stream), ffn_flop),
        "ffn_w2_bias_scatter": gemm_entry(time_reps(ffn2, stream), ffn_flop),
        "ffn_block": time_reps(lambda: (gather(), ffn1(), ffn2()), stream),
    }
    sc_bytes = 5 * tr.eps_c.numel() * 4 + 4 * w.N
    out["stepcache_sw_cfg"] = bw_entry(
        time_reps(lambda: sd.safedit_stepcache_sw_cfg(prev_c, tr.eps_c, prev_u, tr.eps_u, tr.s, 0.5, w.gamma_ctx,
                                                      w.gamma_sens, tr.cfg_out, stream), stream, flush=flush),
        sc_bytes, f"F={tr.eps_c.shape[1]}: {sc_bytes / 1e6:.1f} MB, launch-bound")
    del x, y, xs, h, qkv, w1, w2
    mask = torch.zeros(1, 1, wl.STRESS.N, wl.STRESS.N, dtype=torch.bfloat16, device=dev)
    out["mask_stress"] = bw_entry(
        time_reps(lambda: sd.safedit_mask_is_row_constant(mask, tr.verdict, None, stream), stream, flush=flush),
        mask.numel() * 2, f"[1,1,{wl.STRESS.N},{wl.STRESS.N}] bf16 all-zero mask (removable: read fully)")
    del mask
    # SRSU with kept masks at the stress shape: time per call and slowdown
    # against the same launch with the mask elided
    cases, flop = stress_srsu_cases(sd, dev, stream)
    ms = time_reps_interleaved(cases, stream)
    base = ms["srsu_mask_elided"]["p50"]
    out["kept_mask_stress"] = {
        name: {**t, "tflops": round(flop / (t["p50"] * 1e-3) / 1e12, 1), "vs_elided": round(t["p50"] / base, 3),
               **({"vs_whole_units": round(t["p50"] / ms[name[:-len("_tail_split")]]["p50"], 3)}
                  if name.endswith("_tail_split") else {})}
        for name, t in ms.items()}
    out["kept_mask_stress"]["workload"] = (
        f"B=1, H=32, N={wl.STRESS.N}, d=128, |S|={wl.STRESS.k} (blob scores); padding = trailing 1/8 of the keys "
        "at -inf; bias = [1,1,N,N] N(0,1) in bf16 or f32; each as whole units and tail-balanced; the ten launches "
        "taken in turn within every rep")
    del cases
    torch.cuda.empty_cache()
    out["config_1024"] = measure_1024(sd, dev, stream, flush)
    torch.cuda.empty_cache()
    out["sweep_3072"] = measure_sweep_3072(sd, dev, stream)
    torch.cuda.empty_cache()
    out["guidance_f4096"] = measure_cfg_wide(sd, dev, stream, flush)
    out["workload"] = (f"B={B}, |S|={k} focus rows per batch, D={D}, F={F}; "
                       "synthetic weights N(0,1)/sqrt(fan_in)")
    out["timing"] = "3 warm-ups + 20 CUDA-event reps per entry; p50 (p10 / p90 beside it)"
    if sd.safedit_get_device_status(stream) != 0:
        raise RuntimeError("device status set during the extension measurements")
    return out


def measure_1024(sd, dev, stream, flush):
    """The 1024^2-equivalent configuration (B=2, H=24, N=4096, d=96, L=256
    with 128 valid, |S|=0.3N=1229): every row of the path launched alone on
    its buffers.  Its K/V state (38 MB per tensor) fits in L2, so L2 is
    flushed before every rep."""
    w = wl.W1024
    hbm, bf16_burst, _, src = _peaks()
    tr = Trajectory(w, dev)
    with torch.cuda.stream(stream):
        tr.run(stream)  # fills the split, the state and the scores
    stream.synchronize()
    t = {
        "attn_subset_srsu": time_reps(lambda: tr.attn(
            tr.q, tr.k_state, tr.v_state, tr.idx_s, tr.k, tr.o_state, 1, stream), stream, flush=flush),
        "attn_dense_anchor": time_reps(lambda: tr.attn(
            tr.q, tr.k_state, tr.v_state, None, 0, tr.o_state, 0, stream), stream, flush=flush),
        "attn_dense_anchor_whole_units": time_reps(lambda: sd.safedit_attn_subset(
            tr.q, tr.k_state, tr.v_state, None, 0, None, None, 0.0, tr.o_state, 0, stream), stream, flush=flush),
        "pcsp_score": time_reps(lambda: sd.safedit_pcsp_score(
            tr.q_img, tr.k_txt, tr.valid, tr.content, 0, 0.0, tr.score, stream), stream, flush=flush),
        "cross_attn_probs": time_reps(lambda: sd.safedit_cross_attn_probs(
            tr.q_img, tr.k_txt, tr.valid, 0, 0.0, tr.P, stream), stream, flush=flush),
        "partition_accumulate": time_reps(lambda: sd.safedit_partition_accumulate(
            tr.P, tr.content, tr.score, stream), stream, flush=flush),
        "partition_finalize": time_reps(lambda: sd.safedit_partition_finalize(
            tr.score, w.N, tr.k, tr.idx_s, tr.idx_c, tr.s, stream), stream, flush=flush),
        "scatter_state": time_reps(lambda: sd.safedit_scatter_state(
            [tr.k_s, tr.v_s], [tr.k_state, tr.v_state], tr.idx_s, tr.k, stream), stream, flush=flush),
        "sw_cfg": time_reps(lambda: sd.safedit_sw_cfg(
            tr.eps_c, tr.eps_u, tr.s, w.gamma_ctx, w.gamma_sens, tr.cfg_out, stream), stream, flush=flush),
    }
    for name, flop in (("attn_subset_srsu", tr.flop_srsu), ("attn_dense_anchor", tr.flop_dense),
                       ("attn_dense_anchor_whole_units", tr.flop_dense)):
        tf = flop / (t[name]["p50"] * 1e-3) / 1e12
        t[name].update({"tflops": round(tf, 1), "frac_of_burst": round(tf / bf16_burst, 3)})
    for name, nbytes in tr.bytes.items():
        if name in t:
            gbs = nbytes / (t[name]["p50"] * 1e-3) / 1e9
            t[name].update({"gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)})
    t["workload"] = ("1024^2-equivalent: B=2, H=24, N=4096 (64x64), d=96, L=256 (128 valid), |S|=0.3N=1229; "
                     "L2 flushed before every rep (the 38 MB K/V state would stay in L2)")
    status = sd.safedit_get_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} in the 1024^2 measurements")
    del tr
    return t


def measure_sweep_3072(sd, dev, stream):
    """The 3072^2 sensitive-fraction sweep (B=2, H=24, N=36864, d=96): SRSU
    attention of |S| = rho N rows (the top rho N of the clustered blob scores)
    over all N keys, scattered into the output state, and the dense anchor at
    rho = 1.  Inputs far larger than L2."""
    w = wl.W3072
    _, bf16_burst, bf16_sust, src = _peaks()
    q, k, v = wl.qkv(w, device=dev)
    o = torch.zeros_like(q)
    score = wl.blob_scores(w, device=dev).contiguous()
    out = {}
    for rho in w.rho_sweep:
        kk = wl.k_of(rho, w.N)
        dense = kk == w.N
        idx = None
        if not dense:
            idx = torch.empty(kk, dtype=torch.int32, device=dev)
            sd.safedit_partition_finalize(score, w.N, kk, idx, None, None, stream)
        t = time_reps(lambda: sd.safedit_attn_subset(q, k, v, idx, 0 if dense else kk, None, None, 0.0, o,
                                                     0 if dense else 1, stream), stream, reps=10)
        flop = 4.0 * kk * w.N * w.d * w.B * w.H
        tf = flop / (t["p50"] * 1e-3) / 1e12
        out[f"rho_{float(rho):.1f}"] = {**t, "rows": kk, "dense": dense, "tflop_per_call": round(flop / 1e12, 3),
                                        "tflops": round(tf, 1), "frac_of_burst": round(tf / bf16_burst, 3),
                                        "frac_of_sustained": round(tf / bf16_sust, 3)}
    out["workload"] = "3072^2-equivalent: B=2, H=24, N=36864 (192x192), d=96; 3 warm-ups + 10 reps per point"
    out["peak"] = (f"bf16_tflops burst {bf16_burst}, sustained {bf16_sust} ({src}); the points run right after "
                   "the long trajectory run, under the power cap")
    status = sd.safedit_get_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} in the 3072^2 sweep")
    del q, k, v, o
    return out


def measure_cfg_wide(sd, dev, stream, flush):
    """The guidance combines at a synthetic prediction width F = 4096 over
    N = 25600 tokens (the bandwidth sweep of the launch-bound F = 16 kernels):
    SW-CFG 1.26 GB, StepCache + SW-CFG 2.1 GB per call."""
    w = W
    hbm = _peaks()[0]
    F = 4096
    c, u = wl.cfg_preds(w, device=dev, F=F)
    pc, pu = wl.cfg_preds(w, step=1, device=dev, F=F)
    sv = torch.rand(w.N, device=dev)
    o = torch.empty_like(c)
    res = {}
    for name, fn, nbytes in (
            ("sw_cfg", lambda: sd.safedit_sw_cfg(c, u, sv, w.gamma_ctx, w.gamma_sens, o, stream),
             3 * w.N * F * 4 + 4 * w.N),
            ("stepcache_sw_cfg", lambda: sd.safedit_stepcache_sw_cfg(pc, c, pu, u, sv, 0.5, w.gamma_ctx,
                                                                     w.gamma_sens, o, stream),
             5 * w.N * F * 4 + 4 * w.N)):
        t = time_reps(fn, stream, flush=flush)
        gbs = nbytes / (t["p50"] * 1e-3) / 1e9
        res[name] = {**t, "bytes": nbytes, "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)}
    res["workload"] = f"N={w.N}, F={F} fp32 (synthetic width; the real F=16 is launch-bound)"
    del c, u, pc, pu, o
    return res


def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks (identity when not
    distributed).  Works with NCCL (CUDA device) and gloo (CPU)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() \
            and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(flop_per_rank, n_ranks, max_ms):
    """Weak scaling: every rank runs its own replica, so the job processed
    n_ranks times the per-rank work in the slowest rank's time."""
    return flop_per_rank * n_ranks / (max_ms * 1e-3) / 1e12


def _code_sha(path):
    """sha256 prefix of a C/CUDA source with its comments and whitespace
    removed: equal for two versions that differ only in comments."""
    import hashlib
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256(" ".join(src.split()).encode()).hexdigest()[:16]


def _ncu_traffic():
    """DRAM bytes per SRSU launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu summary, or None when the kernel's code changed
    since those counters were taken (comment-only edits do not count)."""
    p = os.path.join(ROOT, "profiles", "attn_subset_srsu_2560.traffic.json")
    src = os.path.join(ROOT, "spatially_adaptive_dit_b200", "csrc", "attn.cu")
    try:
        with open(p) as f:
            d = json.load(f)
        return d.get("bytes_per_launch") if d.get("attn_cu_code_sha256_16") == _code_sha(src) else None
    except Exception:
        return None


def _packed(tensors, device=None, pin=False):
    """One byte block holding tensors shaped like `tensors` back to back
    (256-byte aligned), and those views of it."""
    sizes = [t.numel() * t.element_size() for t in tensors]
    offs, o = [], 0
    for sz in sizes:
        offs.append(o)
        o += (sz + 255) // 256 * 256
    blk = torch.empty(o, dtype=torch.uint8, device=device, pin_memory=pin)
    views = [blk[off:off + sz].view(t.dtype).view(t.shape) for t, off, sz in zip(tensors, offs, sizes)]
    return blk, views


def run_e2e(tr, stream, args):
    """Same trajectory through the C ABI with host buffers.  Every denoising
    step's inputs are copied from pinned host memory and its guided
    prediction copied back, inside the timed region: on the warm-up step the
    text tensors, on anchor steps the full Q, K, V, and on SRSU steps only the
    fresh S rows -- Q_S, K_S, V_S compact [B,H,k,d] (the projections of an
    SRSU step run on the S rows alone) -- plus eps_c, eps_u every step.  An
    SRSU step is then: scatter K_S, V_S into the cached state, attention of the
    compact Q_S over all N keys, scatter O_S into O_state.  Each step's inputs
    sit back to back in one pinned block and cross the link as one copy (large
    copies reach the link's rate, 70 MB ones do not).  A copy stream runs
    ahead of the compute stream: four SRSU input blocks, and two anchor blocks
    (Q, K, V, predictions) whose K and V then serve as the cached state until
    the next anchor, so an anchor's upload never waits for the step before it;
    events order every buffer reuse.  With three SRSU blocks the upload of the
    fourth step after an anchor waited for the first one's compute, which
    starts only after the anchor's 12 ms: the link idled ~5 ms per anchor."""
    w = tr.w
    NSET = 4
    q_s = tr.q[:, :, : tr.k].contiguous()
    o_s = torch.empty_like(q_s)
    # each step's predictions: both, or (one branch per device) this branch's,
    # gathered with the other device's before the guidance combine
    eps_src = [tr.eps_c, tr.eps_u] if tr.branch is None else [tr.eps_own]
    srsu_src = [q_s, tr.k_s, tr.v_s] + eps_src
    anchor_src = [tr.q, tr.k_full, tr.v_full] + eps_src
    text_src = [tr.q_img, tr.k_txt]
    h_srsu, hv = _packed(srsu_src, pin=True)
    for v, t in zip(hv, srsu_src):
        v.copy_(t)
    h_anchor, hv = _packed(anchor_src, pin=True)
    for v, t in zip(hv, anchor_src):
        v.copy_(t)
    h_text, hv = _packed(text_src, pin=True)
    for v, t in zip(hv, text_src):
        v.copy_(t)
    sets = [_packed(srsu_src, device=tr.dev) for _ in range(NSET)]      # (block, [q_s, k_s, v_s, eps...])
    states = [_packed(anchor_src, device=tr.dev) for _ in range(2)]    # (block, [q, k, v, eps...])
    d_text = _packed(text_src, device=tr.dev)
    out_h = [torch.empty(tr.cfg_out.shape, dtype=tr.cfg_out.dtype, pin_memory=True) for _ in range(NSET)]
    copy_stream = torch.cuda.Stream(device=tr.dev)
    sd = tr.sd
    counts = {"h2d": 0, "d2h": 0}
    freed = [None] * NSET          # per SRSU block: event after the last step that used it
    state_freed = [None, None]     # per anchor block: event after the last step that read it
    text_freed = [None]
    cur_state = [1]                # the anchor block in use (flips at every anchor)

    def trajectory(count):
        with torch.cuda.stream(stream):
            tr.score.zero_()
        for t in range(w.steps):
            anchor = (t % w.period == 0)
            ready = torch.cuda.Event()
            with torch.cuda.stream(copy_stream):
                if t < w.warmup and tr.pcsp_here:
                    if text_freed[0] is not None:
                        copy_stream.wait_event(text_freed[0])
                    d_text[0].copy_(h_text, non_blocking=True)
                    if count:
                        counts["h2d"] += h_text.numel()
                if anchor:
                    cur_state[0] ^= 1
                    if state_freed[cur_state[0]] is not None:
                        copy_stream.wait_event(state_freed[cur_state[0]])  # the previous anchor period
                    blk, src = states[cur_state[0]][0], h_anchor
                else:
                    if freed[t % NSET] is not None:
                        copy_stream.wait_event(freed[t % NSET])  # step t-NSET is done with this block
                    blk, src = sets[t % NSET][0], h_srsu
                blk.copy_(src, non_blocking=True)
                if count:
                    counts["h2d"] += src.numel()
                ready.record(copy_stream)
            aq, k_st, v_st, *a_eps = states[cur_state[0]][1]
            stream.wait_event(ready)
            with torch.cuda.stream(stream):
                if t < w.warmup and tr.pcsp_here:
                    q_img, k_txt = d_text[1]
                    if tr.pcsp == "fused":
                        sd.safedit_pcsp_score(q_img, k_txt, tr.valid, tr.content, 0, 0.0, tr.score, stream)
                    else:
                        sd.safedit_cross_attn_probs(q_img, k_txt, tr.valid, 0, 0.0, tr.P, stream)
                        sd.safedit_partition_accumulate(tr.P, tr.content, tr.score, stream)
                    ev = torch.cuda.Event()
                    ev.record(stream)
                    text_freed[0] = ev
                if t == w.warmup - 1 and tr.reduce_score is not None:
                    tr.reduce_score(tr.score)
                if t == w.warmup - 1 and tr.pcsp_here:
                    sd.safedit_partition_finalize(tr.score, w.N, tr.k, tr.idx_s, tr.idx_c, tr.s, stream)
                if t == w.warmup - 1 and tr.share_split is not None:
                    tr.share_split(tr)
                if t == 0:
                    sd.safedit_mask_is_row_constant(tr.mask, tr.verdict, None, stream)
                if anchor:
                    eps = a_eps
                    tr.attn(aq, k_st, v_st, None, 0, tr.o_state, 0, stream)
                else:
                    qs, ks, vs, *eps = sets[t % NSET][1]
                    sd.safedit_scatter_state([ks, vs], [k_st, v_st], tr.idx_s, tr.k, stream)
                    tr.attn(qs, k_st, v_st, None, 0, o_s, 0, stream)
                    sd.safedit_scatter_state([o_s], [tr.o_state], tr.idx_s, tr.k, stream)
                if tr.branch is None:
                    eps_c, eps_u = eps
                else:  # this branch's prediction as uploaded, the other one from its device
                    tr.eps_own.copy_(eps[0])
                    tr.exchange_eps(tr)
                    eps_c, eps_u = tr.eps_c, tr.eps_u
                g_sens = w.gamma_sens if t >= w.warmup else w.gamma_ctx
                sd.safedit_sw_cfg(eps_c, eps_u, tr.s, w.gamma_ctx, g_sens, tr.cfg_out, stream)
                out_h[t % NSET].copy_(tr.cfg_out, non_blocking=True)
                if count:
                    counts["d2h"] += out_h[t % NSET].numel() * out_h[t % NSET].element_size()
                ev = torch.cuda.Event()
                ev.record(stream)
                if not anchor:
                    freed[t % NSET] = ev
                state_freed[cur_state[0]] = ev

    trajectory(False)
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 5))
    t0 = time.perf_counter()
    for _ in range(n):
        trajectory(True)
    torch.cuda.synchronize()
    ms = (time.perf_counter() - t0) * 1e3 / n
    return {"ms": ms, "h2d": counts["h2d"] // n, "d2h": counts["d2h"] // n}


def oracle_rows(gpu_ms):
    """Every row of the path and of its extensions run by the fp64 oracle, as
    it stands, on the host cores, on a bounded sample of the bench workload;
    the per-call time is extrapolated linearly to the full call (the sample
    and the factor are stated per row) and set beside the GPU's per-call time
    of this run (`gpu_ms`, ms per call by CUDA events)."""
    import numpy as np
    import oracle
    w = W
    out = {}

    def row(name, fn, factor, sample):
        t0 = time.perf_counter()
        fn()
        dt = (time.perf_counter() - t0) * 1e3
        est = dt * factor
        g = gpu_ms.get(name)
        out[name] = {"oracle_ms": round(est, 2), "gpu_ms": None if g is None else round(g, 4),
                     "oracle_over_gpu": None if not g else round(est / g, 1), "sample": sample,
                     "sample_ms": round(dt, 1)}

    q_img, k_txt, valid, content = wl.text(w)
    hs = 2
    P = oracle.cross_attn_probs(q_img[0, :1, :64], k_txt[0, :1], valid[0])  # warm the library
    row("cross_attn_probs", lambda: oracle.cross_attn_probs(q_img[0, :hs], k_txt[0, :hs], valid[0]),
        w.H / hs, f"{hs} of {w.H} heads, all {w.N} rows (x{w.H // hs})")
    P = oracle.cross_attn_probs(q_img[0, :hs], k_txt[0, :hs], valid[0])
    row("partition_accumulate", lambda: oracle.partition_accumulate(P, content), w.H / hs,
        f"{hs} of {w.H} heads (x{w.H // hs})")
    score = wl.blob_scores(wl.Workload("2560 blobs", 2, B=2, H=24, N=w.N, d=96, L=256, n_valid=128,
                                       rho=w.rho, grid=w.grid)).numpy()
    row("partition_finalize", lambda: oracle.partition_select(score, w.k), 1.0,
        f"the full split of N={w.N} (all-pairs rank count)")
    nr = 256
    m = wl.mask(wl.STRESS, "zero", dtype=torch.bfloat16, rows=list(range(nr)))[0, 0]
    row("mask_is_row_constant", lambda: oracle.mask_row_constant(m), wl.STRESS.N / nr,
        f"{nr} of {wl.STRESS.N} rows of the [1,1,{wl.STRESS.N},{wl.STRESS.N}] all-zero mask "
        f"(x{wl.STRESS.N // nr})")
    q, k, v = (t[0, 0].double().numpy() for t in wl.qkv(w))
    ra = 128
    row("attn_dense_anchor", lambda: oracle.attn_subset(q, k, v, np.arange(ra, dtype=np.int32)),
        w.N * w.B * w.H / ra, f"{ra} query rows of one (b,h) over all {w.N} keys (x{w.N * w.B * w.H // ra})")
    row("attn_subset_srsu", lambda: oracle.attn_subset(q, k, v, np.arange(ra, dtype=np.int32)),
        w.k * w.B * w.H / ra, f"{ra} query rows of one (b,h) over all {w.N} keys (x{w.k * w.B * w.H // ra})")
    idx = np.sort(np.random.default_rng(5).choice(w.N, w.k, replace=False)).astype(np.int32)
    ks = wl.fresh_sensitive_kv(w, w.k, step=1)[0][0, 0].view(torch.int16).numpy()
    kst = wl.qkv(w)[1][0, 0].view(torch.int16).numpy()
    row("scatter_state", lambda: oracle.scatter_rows(ks, kst, idx), 2 * w.B * w.H,
        f"one (b,h) slice of K (x{2 * w.B * w.H}: K and V of every slice)")
    ec, eu = wl.cfg_preds(w)
    sv = torch.rand(w.N).numpy()
    row("sw_cfg", lambda: oracle.sw_cfg(ec, eu, sv, w.gamma_ctx, w.gamma_sens), 1.0, f"full [{w.N}, {w.F}]")
    pc, pu = wl.cfg_preds(w, step=1)
    row("stepcache_sw_cfg", lambda: oracle.stepcache_sw_cfg(pc, ec, pu, eu, sv, 0.5, w.gamma_ctx, w.gamma_sens),
        1.0, f"full [{w.N}, {w.F}]")
    D, F = w.D_model, w.D_ff
    w1, b1, w2, b2 = wl.ffn_weights(w)
    x = wl.ffn_states(w)[0][0, :8]
    rf = 8
    row("ffn_block", lambda: oracle.ffn_cached(x, None, w1, b1, w2, b2, np.zeros((rf, D)), act=1),
        w.B * w.k / rf, f"{rf} focus rows (x{w.B * w.k // rf})")
    wq, bq = wl.qkv_proj_weights(w)
    row("qkv_projection_gathered", lambda: oracle.linear_act(x, wq, bq, act=0), w.B * w.k / rf,
        f"{rf} focus rows (x{w.B * w.k // rf})")
    return {"cores": oracle.num_threads(), "kind": "oracle", "rows": out}


def oracle_full_1024(gpu_ms):
    """The 1024^2 configuration's calls run in full (no sampling) by the fp64
    oracle, as it stands, on the host cores, beside the GPU's per-call p50 of
    this run (`gpu_ms`): probabilities and aggregation of the cond branch, the
    split, the SRSU rows and the dense anchor over all 48 slices, the K and V
    scatter of every slice, and the guidance combine."""
    import numpy as np
    import oracle
    w = wl.W1024
    out = {}

    def row(name, fn, what):
        t0 = time.perf_counter()
        r = fn()
        dt = (time.perf_counter() - t0) * 1e3
        g = gpu_ms.get(name)
        out[name] = {"oracle_ms": round(dt, 1), "gpu_ms": None if g is None else round(g, 4),
                     "oracle_over_gpu": None if not g else round(dt / g, 1), "call": what}
        return r

    q_img, k_txt, valid, content = wl.text(w)
    P = row("cross_attn_probs", lambda: oracle.cross_attn_probs(q_img[0], k_txt[0], valid[0]),
            f"[{w.H}, {w.N}, {w.L}] probabilities")
    score = row("partition_accumulate", lambda: oracle.partition_accumulate(P, content), "their aggregation")
    idx_s = row("partition_finalize", lambda: oracle.partition_select(score, w.k), f"the split of N={w.N}")[0]
    q, k, v = (t.double().numpy() for t in wl.qkv(w))
    slices = [(b, h) for b in range(w.B) for h in range(w.H)]
    row("attn_subset_srsu", lambda: [oracle.attn_subset(q[b, h], k[b, h], v[b, h], idx_s) for b, h in slices],
        f"{w.k} rows x {len(slices)} slices over {w.N} keys")
    row("attn_dense_anchor", lambda: [oracle.attn_subset(q[b, h], k[b, h], v[b, h]) for b, h in slices],
        f"all {w.N} rows x {len(slices)} slices (the row-loop routine)")
    ks, vs = (t.view(torch.int16).numpy() for t in wl.fresh_sensitive_kv(w, w.k, step=1))
    kst, vst = (t.view(torch.int16).numpy() for t in wl.qkv(w)[1:])
    row("scatter_state", lambda: [oracle.scatter_rows(src[b, h], dst[b, h], idx_s)
                                  for src, dst in ((ks, kst), (vs, vst)) for b, h in slices],
        f"K and V rows of {len(slices)} slices")
    ec, eu = wl.cfg_preds(w)
    sv = torch.rand(w.N).numpy()
    row("sw_cfg", lambda: oracle.sw_cfg(ec, eu, sv, w.gamma_ctx, w.gamma_sens), f"[{w.N}, {w.F}]")
    return {"cores": oracle.num_threads(), "kind": "oracle", "workload": "1024^2-equivalent, full calls",
            "rows": out}


def cpu_baseline(seconds=12.0, rows=None):
    """The fp64 oracle, as it stands, on the host cores: SRSU attention rows of
    the workload (all k = 7680 sensitive rows of one (b,h) slice per call, over
    all N keys), as many calls as fit in about `seconds` (or exactly `rows`
    rows).  Reported in the metric's unit (TFLOP/s of SRSU attention)."""
    import numpy as np
    import oracle
    w = W
    g = torch.Generator().manual_seed(4321)
    q = torch.randn(w.k, w.d, generator=g).to(torch.bfloat16).double().numpy()
    k = torch.randn(w.N, w.d, generator=g).to(torch.bfloat16).double().numpy()
    v = torch.randn(w.N, w.d, generator=g).to(torch.bfloat16).double().numpy()
    done, dt = 0, 0.0
    chunk = w.k if rows is None else min(rows, w.k)
    t_start = time.perf_counter()
    while True:
        n = chunk if rows is None else min(chunk, rows - done)
        oracle.attn_subset(q, k, v, np.arange(n, dtype=np.int32))
        done += n
        dt = time.perf_counter() - t_start
        if (rows is None and dt >= seconds) or (rows is not None and done >= rows):
            break
        if rows is None and done == chunk and dt < seconds / 64:
            chunk = w.k  # already full slices
    flop = 4.0 * done * w.N * w.d
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done} SRSU query rows ({done / w.k:.2f} slices of k={w.k}) over all N={w.N} keys, "
                      f"d={w.d}, fp64, {dt:.1f} s"}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    import oracle  # noqa: F401
    vals = []
    # calibrate the sample once (about 6 s), then time K steps of that fixed sample
    cal = cpu_baseline(seconds=6.0)
    n_rows = int(cal["sample"].split()[0])
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(rows=n_rows)
        if i >= args.warmup:
            vals.append(r["value"])
    value = statistics.mean(vals)
    ms_per_step = 4.0 * n_rows * W.N * W.d / (value * 1e12) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": W.B, "seq_len": W.N,
                       "parallelism": "host cores (OpenMP)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def stress_srsu_cases(sd, dev, stream):
    """The SRSU launches of the mask-stress workload (B=1, H=32, N=16384,
    d=128, |S|=4915 from the clustered blob scores): mask elided (no mask
    input), kept text-padding key mask (trailing 1/8 of the keys -inf), kept
    non-uniform bias [1,1,N,N] in bf16, both, and the bias in f32; each as
    whole units and tail-balanced (`_tail_split`: 640 units = 4 waves + 48,
    those 48 in 3 key parts).  Returns the launch closures (name -> fn) and
    the flop of one call."""
    w = wl.STRESS
    q, k, v = wl.qkv(w, device=dev)
    o = torch.zeros_like(q)
    score = wl.blob_scores(w, device=dev).contiguous()
    idx = torch.empty(w.k, dtype=torch.int32, device=dev)
    sd.safedit_partition_finalize(score, w.N, w.k, idx, None, None, stream)
    pad = torch.zeros(1, w.N, device=dev)
    pad[:, w.N - w.N // 8:] = float("-inf")
    bias = wl.mask(w, "bias", device=dev)            # [1,1,N,N] bf16
    bias32 = bias.float()                            # the same bias in f32 (1.07 GB)
    att = lambda kp, bb: (lambda: sd.safedit_attn_subset(q, k, v, idx, w.k, kp, bb, 0.0, o, 1, stream))
    nb = sd.safedit_attn_subset_workspace_size(w.B, w.H, w.k, w.N, w.d)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)  # 640 units = 4 waves + 48 split in 3
    att_ws = lambda kp, bb: (lambda: sd.safedit_attn_subset_ws(q, k, v, idx, w.k, kp, bb, 0.0, o, 1, ws, stream))
    cases = {}
    for name, kp, bb in (("srsu_mask_elided", None, None), ("srsu_kept_padding", pad, None),
                         ("srsu_kept_bias", None, bias), ("srsu_kept_padding_and_bias", pad, bias),
                         ("srsu_kept_bias_f32", None, bias32)):
        cases[name] = att(kp, bb)
        cases[name + "_tail_split"] = att_ws(kp, bb)
    return cases, 4.0 * w.k * w.N * w.d * w.B * w.H


def run_stress(args):
    """The mask-path stress workload (B=1, H=32, N=16384, d=128, |S|=4915 from
    the clustered blob scores): SRSU attention with the mask elided (no mask
    input), with a kept text-padding key mask (trailing 1/8 of the keys -inf),
    with a kept non-uniform bf16 bias [1,1,N,N], with both, and with the bias in f32; the row-constant check on
    an all-zero mask (elided: read fully) and on the padding mask (kept: the
    check stops at the first kept row).  Best of `--reps` CUDA-event timings;
    one JSON line per case (not a bench line)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from spatially_adaptive_dit_b200 import safedit as sd
    w = wl.STRESS
    _, bf16_burst, _, src = _peaks()
    stream = torch.cuda.Stream(device=dev)
    cases, flop = stress_srsu_cases(sd, dev, stream)
    zero = wl.mask(w, "zero", device=dev)
    padmask = wl.mask(w, "textpad", device=dev)
    verdict = torch.zeros(1, dtype=torch.int32, device=dev)

    def best(fn):
        times = []
        with torch.cuda.stream(stream):
            for _ in range(args.reps + 1):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                times.append((a, b))
        stream.synchronize()
        return min(a.elapsed_time(b) for a, b in times[1:])

    base = None
    for name, fn in cases.items():
        ms = best(fn)
        base = base or ms
        tf = flop / (ms * 1e-3) / 1e12
        print(json.dumps({"stress": name, "ms": round(ms, 4), "tflops": round(tf, 1),
                          "frac_of_burst": round(tf / bf16_burst, 3), "slowdown": round(ms / base, 3),
                          "peak": f"bf16_tflops {bf16_burst} ({src})"}), flush=True)
    hbm = _peaks()[0]
    for name, m in (("mask_check_elided_zero", zero), ("mask_check_kept_padding", padmask)):
        ms = best(lambda: sd.safedit_mask_is_row_constant(m, verdict, None, stream))
        gbs = m.numel() * 2 / (ms * 1e-3) / 1e9
        print(json.dumps({"stress": name, "ms": round(ms, 4), "verdict": int(verdict.item()),
                          "gbs_if_read_fully": round(gbs, 1), "frac_hbm_if_read_fully": round(gbs / hbm, 3)}),
              flush=True)
    status = sd.safedit_get_device_status(stream)
    if status != 0:
        print(json.dumps({"stress": "status", "status": status}))
        sys.exit(3)


def run_sweep(args):
    """The 3072^2 sensitive-fraction sweep (B=2, H=24, N=36864, d=96): SRSU
    attention of |S| = rho N gathered rows over all N keys, scattered into the
    output state, for rho in {0.1, 0.2, 0.3, 0.5}, and the dense anchor
    (rho = 1).  Best of `--reps` CUDA-event timings per point; one JSON line
    per point (not a bench line)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from spatially_adaptive_dit_b200 import safedit as sd
    w = wl.W3072
    _, bf16_burst, bf16_sust, src = _peaks()
    q, k, v = wl.qkv(w, device=dev)
    o = torch.zeros_like(q)
    stream = torch.cuda.Stream(device=dev)
    g = torch.Generator().manual_seed(3072)
    perm = torch.randperm(w.N, generator=g)
    for rho in w.rho_sweep:
        kk = wl.k_of(rho, w.N)
        dense = kk == w.N
        idx = None if dense else torch.sort(perm[:kk]).values.to(torch.int32).to(dev)
        times = []
        with torch.cuda.stream(stream):
            for _ in range(args.reps + 1):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                sd.safedit_attn_subset(q, k, v, idx, 0 if dense else kk, None, None, 0.0, o,
                                       0 if dense else 1, stream)
                b.record(stream)
                times.append((a, b))
        stream.synchronize()
        ms = min(a.elapsed_time(b) for a, b in times[1:])
        flop = 4.0 * kk * w.N * w.d * w.B * w.H
        tf = flop / (ms * 1e-3) / 1e12
        status = sd.safedit_get_device_status(stream)
        print(json.dumps({"sweep": "3072", "rho": float(rho), "rows": kk, "dense": dense, "ms": round(ms, 4),
                          "tflops": round(tf, 1), "frac_of_burst": round(tf / bf16_burst, 3),
                          "peak": f"bf16_tflops {bf16_burst} ({src})", "status": status}), flush=True)
        if status != 0:
            sys.exit(3)


def run_only(args):
    """One kernel of the path in isolation, `--reps` times on the bench
    workload's buffers (`--config` picks another configuration's; the target
    of ncu captures and quick timing).  Prints per-launch CUDA-event times;
    not a bench line."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from spatially_adaptive_dit_b200 import safedit as sd
    w = {"2560": W, "1024": wl.W1024, "3072": wl.W3072}[args.config]
    tr = Trajectory(w, dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        sd.safedit_cross_attn_probs(tr.q_img, tr.k_txt, tr.valid, 0, 0.0, tr.P, stream)
        sd.safedit_partition_accumulate(tr.P, tr.content, tr.score, stream)
        sd.safedit_partition_finalize(tr.score, w.N, tr.k, tr.idx_s, tr.idx_c, tr.s, stream)
    stream.synchronize()
    extra = {}
    if args.only in ("cfg", "stepcache") and args.cfg_f != w.F:
        # bandwidth sweep of the guidance combine at a wider prediction (synthetic)
        tr.eps_c, tr.eps_u = wl.cfg_preds(w, device=dev, F=args.cfg_f)
        tr.cfg_out = torch.empty_like(tr.eps_c)
        tr.bytes["sw_cfg"] = 3 * w.N * args.cfg_f * 4 + 4 * w.N
    if args.only == "stepcache":  # predictions of the previous full step: distinct tensors
        extra["prev_c"], extra["prev_u"] = wl.cfg_preds(w, step=1, device=dev, F=tr.eps_c.shape[1])
    if args.only == "mask":
        extra["mask"] = torch.zeros(1, 1, wl.STRESS.N, wl.STRESS.N, dtype=torch.bfloat16, device=dev)
    ffn_flop = 2 * w.B * tr.k * w.D_model * w.D_ff  # one projection of the cached FFN
    if args.only in ("ffn1", "ffn2", "ffn", "qkv"):
        # SkipSparse FFN caching on the focus rows: gather, W1 (+b1, GELU), W2 (+b2) scattered
        w1, b1, w2, b2 = (t.to(dev) for t in wl.ffn_weights(w))
        x, y = (t.to(dev) for t in wl.ffn_states(w))
        xs = torch.empty(w.B, 1, tr.k, w.D_model, dtype=torch.bfloat16, device=dev)
        h = torch.empty(w.B, tr.k, w.D_ff, dtype=torch.bfloat16, device=dev)
        sd.safedit_gather_rows([x.view(w.B, 1, w.N, w.D_model)], [xs], tr.idx_s, tr.k, stream)
        xs3 = xs.view(w.B, tr.k, w.D_model)
        extra["ffn1"] = lambda: sd.safedit_gemm_bias_act(xs3, w1, b1, 1, None, h, stream)
        extra["ffn2"] = lambda: sd.safedit_gemm_bias_act(h, w2, b2, 0, tr.idx_s, y, stream)
        wqkv, bqkv = (t.to(dev) for t in wl.qkv_proj_weights(w))
        qkv = torch.empty(w.B, tr.k, 3 * w.D_model, dtype=torch.bfloat16, device=dev)
        extra["qkv"] = lambda: sd.safedit_gemm_bias_act(xs3, wqkv, bqkv, 0, None, qkv, stream)

        def ffn_block():
            sd.safedit_gather_rows([x.view(w.B, 1, w.N, w.D_model)], [xs], tr.idx_s, tr.k, stream)
            extra["ffn1"]()
            extra["ffn2"]()
        extra["ffn"] = ffn_block
    fns = {
        "srsu": (lambda: sd.safedit_attn_subset(tr.q, tr.k_state, tr.v_state, tr.idx_s, tr.k, None, None,
                                                0.0, tr.o_state, 1, stream), tr.flop_srsu, None),
        "anchor": (lambda: sd.safedit_attn_subset(tr.q, tr.k_state, tr.v_state, None, 0, None, None, 0.0,
                                                  tr.o_state, 0, stream), tr.flop_dense, None),
        # the tail-balanced entry point as the trajectory calls it (whole units,
        # key-range parts and their merge where the plan splits)
        "srsu_ws": (lambda: tr.attn(tr.q, tr.k_state, tr.v_state, tr.idx_s, tr.k, tr.o_state, 1, stream),
                    tr.flop_srsu, None),
        "anchor_ws": (lambda: tr.attn(tr.q, tr.k_state, tr.v_state, None, 0, tr.o_state, 0, stream),
                      tr.flop_dense, None),
        "xattn": (lambda: sd.safedit_cross_attn_probs(tr.q_img, tr.k_txt, tr.valid, 0, 0.0, tr.P, stream),
                  None, tr.bytes["cross_attn_probs"]),
        "accumulate": (lambda: sd.safedit_partition_accumulate(tr.P, tr.content, tr.score, stream), None,
                       tr.bytes["partition_accumulate"]),
        "pcsp": (lambda: sd.safedit_pcsp_score(tr.q_img, tr.k_txt, tr.valid, tr.content, 0, 0.0, tr.score,
                                               stream), None, w.H * w.N * w.d * 2 + w.H * w.L * w.d * 2),
        "finalize": (lambda: sd.safedit_partition_finalize(tr.score, w.N, tr.k, tr.idx_s, tr.idx_c, tr.s,
                                                           stream), None, None),
        "scatter": (lambda: sd.safedit_scatter_state([tr.k_s, tr.v_s], [tr.k_state, tr.v_state], tr.idx_s,
                                                     tr.k, stream), None, tr.bytes["scatter_state"]),
        "cfg": (lambda: sd.safedit_sw_cfg(tr.eps_c, tr.eps_u, tr.s, w.gamma_ctx, w.gamma_sens, tr.cfg_out,
                                          stream), None, tr.bytes["sw_cfg"]),
        "mask": (lambda: sd.safedit_mask_is_row_constant(extra["mask"], tr.verdict, None, stream), None,
                 wl.STRESS.N * wl.STRESS.N * 2),
        "stepcache": (lambda: sd.safedit_stepcache_sw_cfg(extra["prev_c"], tr.eps_c, extra["prev_u"], tr.eps_u,
                                                          tr.s, 0.5, w.gamma_ctx, w.gamma_sens, tr.cfg_out,
                                                          stream),
                      None, 5 * tr.eps_c.numel() * 4 + 4 * w.N),
        "ffn1": (lambda: extra["ffn1"](), ffn_flop, None),
        "ffn2": (lambda: extra["ffn2"](), ffn_flop, None),
        "ffn": (lambda: extra["ffn"](), 2 * ffn_flop, None),
        "qkv": (lambda: extra["qkv"](), 3 * ffn_flop / w.ffn_mult, None),
    }
    fn, flop, nbytes = fns[args.only]
    times = []
    flush = L2Flush(dev) if args.flush else None
    with torch.cuda.stream(stream):
        for i in range(args.reps):
            if flush is not None:
                flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            times.append((a, b))
    stream.synchronize()
    ms = [a.elapsed_time(b) for a, b in times]
    status = sd.safedit_get_device_status(stream)
    out = {"only": args.only, "reps": args.reps, "ms": [round(x, 4) for x in ms], "status": status,
           "l2_flushed": bool(args.flush)}
    if args.only in ("cfg", "stepcache"):
        out["F"] = args.cfg_f
    best = min(ms[1:] if len(ms) > 1 else ms)
    if flop:
        out["tflops_best"] = round(flop / (best * 1e-3) / 1e12, 1)
    if nbytes:
        out["gbs_best"] = round(nbytes / (best * 1e-3) / 1e9, 1)
    print(json.dumps(out), flush=True)
    if status != 0:
        sys.exit(3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads", "cfg"],
                    help="N > 1: independent replicas (default, weak scaling), one generation split by heads "
                         "(strong scaling; the PCSP score is all-reduced once), or, on 2 GPUs, one generation "
                         "split by guidance branch (the split broadcast once, the predictions gathered every step)")
    ap.add_argument("--pcsp", default="fused", choices=["fused", "unfused"],
                    help="PCSP warm-up in the timed trajectory: the fused score kernel (default) or the "
                         "probabilities kernel followed by the aggregation")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None,
                    choices=["srsu", "anchor", "srsu_ws", "anchor_ws", "xattn", "accumulate", "pcsp", "finalize", "scatter", "cfg",
                             "stepcache", "mask", "ffn1", "ffn2", "ffn", "qkv", "sweep", "stress"],
                    help="run one kernel of the path in isolation (profiling target)")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--config", default="2560", choices=["2560", "1024", "3072"],
                    help="with --only: the configuration whose buffers the kernel runs on (3072: rho = 0.3)")
    ap.add_argument("--flush", action="store_true", help="--only: flush L2 before every rep (outside the events)")
    ap.add_argument("--cfg-f", type=int, default=W.F, help="prediction width for --only cfg")
    args = ap.parse_args()
    if args.only == "sweep":
        run_sweep(args)
        return
    if args.only == "stress":
        run_stress(args)
        return
    if args.only:
        run_only(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
