#!/usr/bin/env python
"""Benchmark of one batched block-Shampoo (DASH-style) optimizer step on B200.

Default workload: a ~1B Llama-shaped parameter set (24 layers, d=2048, SwiGLU
MLP 2048x5632 x3, embedding and head 32000x2048), fp32 gradients N(0, 1e-2)
with a per-row LogNormal(0, 1) scale, block size B=1024, every step
preconditioned: factor EMA, 10 power-iteration products from 32 starts,
Newton-DB 14 + 14 iterations (or Chebyshev), preconditioning, Adam graft and
update.  Inputs are synthetic (seeded) and resident in HBM; the working set
(~100 GB) is far larger than L2, so no L2 flush is needed between steps.

One JSON line on rank 0: the step time (ms, lower is better), the roofline of
the dominant kernel (the tensor-core GEMM, per-launch CUDA-event durations
measured inside the timed region), the root-stage TFLOP/s as a fraction of the
dense TF32 peak, an end-to-end figure through the C ABI with host buffers, the
SM clocks sampled during the timed region, and the float64 oracle timed on the
host cores on a bounded sample of the same workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload llama1b|gpt2|spiked512|roots256|mixed]

For N > 1 (torchrun, one process per GPU) the parameters are shared out by
greedy ownership (decreasing root cost, least-loaded rank first); each rank
runs the step for the blocks of the parameters it owns and one NCCL
all-gather per step gives every rank all updated parameters (strong scaling:
the workload is fixed).  The step time is the max over ranks.  The standalone
roots workload runs one replica per rank.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")

# DRAM bytes (read + write) per executed tensor-core flop of the GEMM, by
# (kernel, block size, solver): from an ncu capture of every launch of three
# steps of the mixed-shape B=1024 workload (24 factors of 1024, Newton-DB
# 14 + 14): 59.82 GB over 3.69e13 executed flops.  Each launch reads and writes
# its problems' split matrices about once, so a launch's traffic grows in
# proportion to the problems, and executed flops, it covers; the roofline's
# per-launch traffic scales this ratio by those flops.
GEMM_DRAM_BYTES_PER_FLOP = {("gemm_wide_kernel", 1024, "ndb"): 1.622e-3}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="llama1b",
                   choices=["llama1b", "gpt2", "spiked512", "roots256", "mixed"])
    p.add_argument("--block", type=int, default=None, help="override the block size")
    p.add_argument("--solver", default="ndb", choices=["ndb", "cheb", "cn", "cn16"],
                   help="Newton-DB, Chebyshev, coupled Newton (split products) or coupled Newton in fp16")
    p.add_argument("--cn-iters", type=int, default=16)
    p.add_argument("--iters", type=int, default=None, help="Newton-DB iterations per stage")
    p.add_argument("--degree", type=int, default=16)
    p.add_argument("--n", type=int, default=256, help="matrices in the standalone-roots workload")
    p.add_argument("--root-every", type=int, default=1,
                   help="recompute roots every F-th step and reuse them in between (default: every step)")
    p.add_argument("--scaling", default="spectral", choices=["spectral", "frobenius"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--graph", action="store_true",
                   help="standalone roots workload: capture one root call in a CUDA graph and time its replays")
    p.add_argument("--e2e-groups", type=int, default=4,
                   help="parameter groups of the host-buffer step on one GPU (copies overlap the other "
                        "groups' work); 1: upload, step and download one after the other")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

def workload_spec(args):
    from matrix_inverse_roots_stack_b200 import workloads as wl
    if args.workload == "llama1b":
        spec = dict(shapes=wl.llama_1b_shapes(), B=1024, grad="lognormal", iters=14,
                    desc="llama-1b-shaped param set (24 layers, d=2048, SwiGLU 2048x5632 x3, "
                         "embed+head 32000x2048), fp32 grads N(0,1e-2) x row LogNormal(0,1)")
    elif args.workload == "gpt2":
        spec = dict(shapes=wl.gpt2_124m_shapes(), B=512, grad="gauss", iters=14,
                    desc="gpt2-124m-shaped param set (12 layers, d=768, QKV 768x2304, attn-out, "
                         "MLP 768x3072/3072x768, wte 50257x768, wpe 1024x768), fp32 grads N(0,1e-2)")
    elif args.workload == "spiked512":
        spec = dict(shapes=[(512, 512)], B=128, grad="spiked", iters=8,
                    desc="single 512x512 fp32 weight, gradient N(0,1) + rank-8 spike (scale 10)")
    elif args.workload == "mixed":
        spec = dict(shapes=wl.mixed_shapes(), B=1024, grad="student", iters=14,
                    desc="mixed shapes 1024x4096, 4096x1024, 2048x2048, Student-t(3) grads")
    else:
        spec = dict(shapes=None, B=256, grad=None, iters=14, n=args.n,
                    desc=f"standalone inverse 4th roots: {args.n} SPD blocks, A = G G^T/1024 + 1e-6 I, "
                         "singular values of G decaying as 1/k")
    if args.block:
        spec["B"] = args.block
    if args.iters:
        spec["iters"] = args.iters
    return spec


def make_grads(spec, device, seed=0):
    import torch
    from matrix_inverse_roots_stack_b200 import workloads as wl
    if spec["grad"] == "lognormal":
        return wl.torch_gaussian_gradients(spec["shapes"], device, std=0.1, seed=seed, row_lognormal_sigma=1.0)
    if spec["grad"] == "gauss":
        return wl.torch_gaussian_gradients(spec["shapes"], device, std=0.1, seed=seed)
    if spec["grad"] == "student":
        return wl.torch_student_t_gradients(spec["shapes"], device, nu=3.0, seed=seed)
    if spec["grad"] == "spiked":
        return [torch.from_numpy(wl.spiked_gradient(512, 512, rank=8, scale=10.0, seed=seed)).to(device)]
    raise ValueError(spec["grad"])


def block_sizes(shapes, B):
    out = []
    for (r, c) in shapes:
        for r0 in range(0, r, B):
            for c0 in range(0, c, B):
                out.append((min(B, r - r0), min(B, c - c0)))
    return out


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        note = None
        if not rows:
            # the timed region ended before the sampler's first reading: take
            # one reading now, right after it
            try:
                q = subprocess.run(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                    "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
                rows = [[x.strip() for x in line.split(",")] for line in q.stdout.splitlines()
                        if len(line.split(",")) >= 9]
                note = "timed region shorter than the sampler's start-up: one reading right after it"
            except (OSError, subprocess.SubprocessError):
                rows = []
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
               "reasons": reasons, "samples": len(rows)}
        if note:
            out["note"] = note
        return out


# --------------------------------------------------------------------------
# CPU baseline / reference arm: the float64 oracle on a bounded sample
# --------------------------------------------------------------------------

# Blocks of the workload the oracle is timed on (the first parameters, in
# order, until at least this many blocks): one fixed sample, used by both the
# cpu_baseline leg and the reference arm, of about 5-15 s of CPU work.
ORACLE_SAMPLE_BLOCKS = {"llama1b": 40, "gpt2": 60, "spiked512": 16, "mixed": 12, "roots256": 4}


def oracle_sample(spec, args, seed=0):
    """Time the oracle step on a fixed sample of the workload's blocks
    (ORACLE_SAMPLE_BLOCKS); returns (ms per full step extrapolated by block
    count, description, threads)."""
    import numpy as np
    from oracle import step as ostep, roots
    from matrix_inverse_roots_stack_b200 import workloads as wl
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        threads = os.cpu_count()
    B = spec["B"]
    iters = spec["iters"]
    hp = ostep.HParams(block_size=B, ndb_iters1=iters, ndb_iters2=iters,
                       solver={"ndb": "ndb", "cheb": "cheb"}.get(args.solver, "cn"), cheb_degree=args.degree,
                       cn_iters=args.cn_iters)
    V0 = wl.pi_start_vectors(B, 32, seed=0).astype(np.float64)
    target = ORACLE_SAMPLE_BLOCKS[args.workload]
    if spec["shapes"] is None:  # standalone roots: time per matrix
        nmat = spec.get("n", 256)
        A, _, _ = wl.spd_stack_decaying(n=min(target, nmat), b=B, seed=seed)
        t0 = time.perf_counter()
        done = 0
        for i in range(A.shape[0]):
            ostep.inverse_fourth_root(A[i].astype(np.float64), V0, hp)  # power iteration + the solver
            done += 1
        dt = time.perf_counter() - t0
        return (dt / done * nmat * 1e3, f"{done} of {nmat} matrices ({B}x{B}), extrapolated x{nmat / done:.1f}",
                threads)
    shapes = spec["shapes"]
    total_blocks = len(block_sizes(shapes, B))
    rng = np.random.default_rng(seed)
    t0 = time.perf_counter()
    done_blocks, used = 0, []
    for (r, c) in shapes:
        G = rng.standard_normal((r, c)) * 0.1
        th = np.zeros((r, c))
        state = ostep.init_state([(r, c)], hp)
        ostep.shampoo_step([th], [G], state, hp, V0)
        done_blocks += len(block_sizes([(r, c)], B))
        used.append(f"{r}x{c}")
        if done_blocks >= target:
            break
    dt = time.perf_counter() - t0
    frac = total_blocks / done_blocks
    return (dt * frac * 1e3, f"oracle step (level 2, eigh) on parameters {', '.join(used)} = {done_blocks} of "
            f"{total_blocks} blocks, extrapolated x{frac:.1f} by block count", threads)


def arm_config(args, spec, world):
    """The workload description both arms report (identical dicts)."""
    cfg = {"workload": spec["desc"], "block_size": spec["B"], "solver": args.solver,
           "iters_per_stage": spec["iters"] if args.solver == "ndb" else None,
           "cheb_degree": args.degree if args.solver == "cheb" else None,
           "cn_iters": args.cn_iters if args.solver in ("cn", "cn16") else None,
           "scale_estimate": ("power iteration, 10 products x 32 starts" if args.scaling == "spectral"
                              else "Frobenius norm"),
           "roots_every_steps": max(1, args.root_every),
           "l2": ("working set far larger than the 126 MB L2 (no flush needed)" if spec["B"] >= 512 and
                  spec["shapes"] is not None else "small working set, no L2 flush between steps (not a headline)"),
           "parallelism": ("one GPU" if world == 1 else
                           f"replicas x{world}" if spec["shapes"] is None else
                           f"sharded x{world}: greedy parameter ownership by root cost, "
                           "NCCL all-gather of the updated parameters")}
    if spec["shapes"] is not None:
        nb = len(block_sizes(spec["shapes"], spec["B"]))
        cfg.update({"n_params": len(spec["shapes"]), "n_blocks": nb, "n_factors": 2 * nb})
    else:
        cfg["n_matrices"] = spec["n"]
    return cfg


def run_reference(args, spec, rank):
    if rank != 0:
        return
    per_step = []
    for i in range(args.warmup + args.steps):
        ms, sample, threads = oracle_sample(spec, args)
        if i >= args.warmup:
            per_step.append(ms)
    ms = statistics.median(per_step)
    line = {"impl": "reference", "metric": "Shampoo optimizer step ms", "value": round(ms, 3), "unit": "ms",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": arm_config(args, spec, args.gpus),
            "cpu_baseline": {"value": round(ms, 3), "unit": "ms", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(ms, 3), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def main():
    args = parse_args()
    spec = workload_spec(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, spec, rank)
        return 0

    import torch
    import torch.distributed as dist
    from matrix_inverse_roots_stack_b200 import binding as bd, build, workloads as wl
    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    B = spec["B"]
    iters = spec["iters"]
    solver = {"ndb": bd.SOLVER_NEWTON_DB, "cheb": bd.SOLVER_CHEBYSHEV}.get(args.solver, bd.SOLVER_COUPLED_NEWTON)
    cn16 = args.solver == "cn16"
    stream = torch.cuda.current_stream()

    if spec["shapes"] is None:
        # standalone roots workload
        nmat = spec["n"]
        A, _, _ = wl.spd_stack_decaying(n=nmat, b=B, seed=0)
        At = torch.from_numpy(A).to(dev)
        X = torch.empty_like(At)
        lam = torch.empty(nmat, dtype=torch.float32, device=dev)
        v0 = torch.from_numpy(wl.pi_start_vectors(B, 32, seed=0)).to(dev)
        need = bd.inv_root_workspace_bytes(nmat, B, solver)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)

        def step_fn():
            if solver == bd.SOLVER_NEWTON_DB:
                bd.inv_root_newton_db(At, v0, iters, iters, 0.0, 10, X, lam, ws)
            elif solver == bd.SOLVER_COUPLED_NEWTON:
                bd.inv_root_coupled_newton(At, v0, args.cn_iters, cn16, 0.0, 10, X, lam, ws)
            else:
                bd.inv_root_chebyshev(At, v0, args.degree, 1e-3, 0.0, 10, X, lam, ws)
        n_factors, factor_sizes = nmat, [B] * nmat
        ctx_info = {}
        e2e_fn = None
        eager_fn = step_fn
    else:
        grads = make_grads(spec, dev, seed=0)
        params = [torch.randn(g.shape, device=dev) * 0.02 for g in grads]
        hp = bd.make_hparams(block_size=B, solver=solver, ndb_iters1=iters, ndb_iters2=iters,
                             cheb_degree=args.degree, root_every=args.root_every, cn_iters=args.cn_iters,
                             cn_fp16=1 if cn16 else 0,
                             scaling=bd.SCALING_FROBENIUS if args.scaling == "frobenius" else bd.SCALING_SPECTRAL)
        v0 = torch.from_numpy(wl.pi_start_vectors(B, 32, seed=0)).to(dev)
        # one rank per GPU: greedy ownership of the parameters, each rank steps
        # its own and one all-gather per step distributes the results
        from matrix_inverse_roots_stack_b200 import distributed as sd
        sharded = sd.ShardedShampoo(params, grads, B, make_local=lambda ps, gs: bd.Shampoo(ps, gs, hp=hp, v0=v0))
        live = {"sharded": sharded}
        g_off = [0]
        for g in grads:
            g_off.append(g_off[-1] + g.numel())
        opt = sharded.local
        if opt is None:
            raise SystemExit(f"rank {rank} owns no parameter: use fewer GPUs for this workload")
        owned_shapes = [tuple(params[i].shape) for i in sharded.owned]
        bsz = block_sizes(owned_shapes, B)
        factor_sizes = [s for pair in bsz for s in pair]
        n_factors = opt.n_factors
        ctx_info = {"rank0_owned_params": len(sharded.owned), "rank0_n_factors": opt.n_factors,
                    "workspace_gb": round(opt.ws.numel() / 1e9, 2)}

        def step_fn():
            live["sharded"].step()
        eager_fn = step_fn

        def e2e_fn(host_g, host_p):
            # the same step through the C ABI with host buffers: upload the
            # step's gradients from pinned memory, step, read the parameters back
            if "pipe" in live:  # one GPU: copies overlapped with the other groups' work
                live["pipe"].step(live["hg"], live["hp"])
                return
            # a rank reads only the gradients of the parameters it owns
            sh = live["sharded"]
            for i in sh.owned:
                n = grads[i].numel()
                grads[i].view(-1).copy_(host_g[g_off[i]:g_off[i] + n], non_blocking=True)
            sh.step()
            off = 0
            for p in params:
                n = p.numel()
                host_p[off:off + n].copy_(p.view(-1), non_blocking=True)
                off += n

    # ---------------- warm-up
    for _ in range(args.warmup):
        step_fn()
    torch.cuda.synchronize()
    if spec["shapes"] is not None:
        rc, flags = opt.status()
        if rc != 0:
            print(f"[bench] warning: status {bd.strerror(rc)} (flags {flags})", file=sys.stderr)

    graph = None
    if args.graph and spec["shapes"] is None:
        # one root call captured after the eager warm-up; the timed region
        # replays it (kernels inside a graph record no profiling events, so
        # the per-launch figures come from eager calls after the timed region)
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            eager_fn()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        step_fn = graph.replay
        ctx_info["cuda_graph"] = "timed steps replay one captured root call; per-launch figures from eager calls"

    # ---------------- timed region (no per-launch events: profiling off)
    bd.profile_reset()
    bd.profile_enable(False)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step_fn()
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    launches = bd.profile_read()["launches"]  # kernels launched in the timed steps (eager calls)
    ms = t_start.elapsed_time(t_stop) / args.steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    # ---------------- instrumented pass: the next steps again, with a CUDA
    # event pair around every GEMM launch and stage (per-launch roofline and
    # stage times; its step time is reported beside the headline)
    prof_steps = min(args.steps, 3)
    bd.profile_reset()
    bd.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    p_start = torch.cuda.Event(enable_timing=True)
    p_stop = torch.cuda.Event(enable_timing=True)
    p_start.record(stream)
    for _ in range(prof_steps):
        eager_fn()
    p_stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    bd.profile_enable(False)
    prof = bd.profile_read()
    prof_ms = p_start.elapsed_time(p_stop) / prof_steps
    if graph is not None:
        launches = prof["launches"] * args.steps // prof_steps  # a replay launches what an eager call does

    # ---------------- end to end through host buffers
    e2e = None
    if e2e_fn is not None and not args.no_e2e:
        n_g = sum(g.numel() for g in grads)
        n_p = sum(p.numel() for p in params)
        try:
            host_g = torch.empty(n_g, dtype=torch.float32, pin_memory=True)
            host_p = torch.empty(n_p, dtype=torch.float32, pin_memory=True)
            off = 0
            for g in grads:
                host_g[off:off + g.numel()].copy_(g.view(-1).cpu())
                off += g.numel()
            if world == 1 and args.e2e_groups > 1:
                # the pipelined host-buffer step keeps its own device state: release
                # the device-resident optimizer first
                from matrix_inverse_roots_stack_b200.pipeline import HostPipelinedShampoo
                live.clear()
                opt = sharded = None
                torch.cuda.empty_cache()
                pipe = HostPipelinedShampoo([tuple(p.shape) for p in params], hp=hp, v0=v0, device=dev,
                                            groups=args.e2e_groups)
                hg, hpl, off = [], [], 0
                for p in params:
                    n = p.numel()
                    hg.append(host_g[off:off + n].view(p.shape))
                    hpl.append(host_p[off:off + n].view(p.shape))
                    host_p[off:off + n].copy_(p.view(-1).cpu())
                    off += n
                pipe.load_params(hpl)
                live.update(pipe=pipe, hg=hg, hp=hpl)
                e2e_info = {"groups": len(pipe.groups), "overlap": "uploads, steps and downloads of groups "
                            "on three streams"}
            else:
                e2e_info = {"groups": 1, "overlap": "none"}
            e2e_fn(host_g, host_p)
            torch.cuda.synchronize()
            barrier()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                e2e_fn(host_g, host_p)
            e1.record(stream)
            torch.cuda.synchronize()
            e_ms = e0.elapsed_time(e1) / args.steps
            if world > 1:
                t = torch.tensor([e_ms], device=dev)
                dist.all_reduce(t, op=dist.ReduceOp.MAX)
                e_ms = float(t.item())
            h2d = 4 * (n_g if world == 1 else sum(grads[i].numel() for i in sharded.owned))
            e2e = {"value": round(e_ms, 3), "unit": "ms", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": 4 * n_p, **e2e_info}
            del host_g, host_p
        except RuntimeError as exc:
            e2e = {"value": None, "unit": "ms", "error": str(exc)[:200]}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---------------- roofline of the dominant kernel (a split-fp16 GEMM)
    peaks, peak_kind = load_peaks()
    tensor_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    kernels = {"gemm_wide_kernel": prof["gemm_wide"], "gemm_split_kernel": prof["gemm"],
               "ndb_fused_kernel": prof["ndb_fused"]}

    def kernel_line(ms_, n_, fl_):
        avg = ms_ / max(n_, 1)
        # executed fp16 MMA flops as the library records them (3 per useful product, 1 in fp16 mode)
        ach = (fl_ / max(n_, 1)) / (avg * 1e-3) / 1e12 if n_ else None
        return avg, ach

    name = max(kernels, key=lambda k: kernels[k][0])
    g_ms, g_n, g_flops = kernels[name]
    avg_ms, achieved = kernel_line(g_ms, g_n, g_flops)
    bpf = GEMM_DRAM_BYTES_PER_FLOP.get((name, B, args.solver))
    traffic = round(bpf * g_flops / g_n) if (bpf and g_n) else None
    roofline = {"kernel": name, "bound": "tensor",
                "achieved": round(achieved, 1) if achieved else None, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": round(achieved / tensor_peak, 4) if achieved else None,
                "traffic": traffic, "traffic_unit": "bytes per launch (ncu DRAM read+write, scaled by executed flops)"
                if traffic else None, "peak_kind": f"{peak_kind} bf16/fp16 dense, sustained",
                "launches": g_n, "avg_launch_ms": round(avg_ms, 4),
                "share_of_step": round(g_ms / (prof_ms * prof_steps), 4),
                "measured_in": f"instrumented pass of {prof_steps} steps after the timed ones "
                               f"({round(prof_ms, 3)} ms per step with the events)",
                "gemm_kernels": {k: {"launches": v[1], "ms": round(v[0] / prof_steps, 3),
                                     "tflops_executed": round(kernel_line(*v)[1], 1) if v[1] else None}
                                 for k, v in kernels.items()},
                "wide_kernel_regs": prof.get("wide_regs")}

    # ---------------- root-stage TFLOP/s vs dense TF32 peak
    s_ms = prof["solver"][0] + prof["power_iteration"][0]
    if graph is not None:
        s_ms = ms * prof_steps  # the standalone step is the root stage (graph replays, no events)
    if args.solver == "ndb":
        gemms = 2 * (3 * iters - 3)            # both stages, first-iteration and last-iteration savings
    elif args.solver in ("cn", "cn16"):
        gemms = 4 * (args.cn_iters - 1) + 1    # C^2, C^4, C^4 M, X C; the last iteration only X C
    else:
        gemms = args.degree - 1
    padded = 2.0 * B ** 3 * gemms * n_factors
    unpadded = sum(2.0 * b ** 3 * gemms for b in factor_sizes)
    tf32_peak = tensor_peak / 2.0
    # instrumented steps are W+K+1 .. W+K+P; roots are computed on steps with (t-1) % f == 0
    every = max(1, args.root_every) if spec["shapes"] is not None else 1
    t0_step = args.warmup + args.steps
    root_steps = sum(1 for t in range(t0_step + 1, t0_step + prof_steps + 1) if (t - 1) % every == 0)
    inverse_root = None
    if root_steps and s_ms > 0:
        root_s = s_ms * 1e-3 / root_steps
        inverse_root = {"ms_per_root_step": round(root_s * 1e3, 3), "root_steps_profiled": root_steps,
                        "tflops": round(padded / root_s / 1e12, 1),
                        "tflops_unpadded": round(unpadded / root_s / 1e12, 1),
                        "tf32_peak_tflops": tf32_peak,
                        "frac_of_tf32_peak": round(padded / root_s / 1e12 / tf32_peak, 4),
                        "frac_of_tf32_peak_unpadded": round(unpadded / root_s / 1e12 / tf32_peak, 4),
                        "peak_kind": f"{peak_kind}: bf16 sustained x 0.5 (nominal TF32/BF16 ratio)"}
    stages = {k: round(v[0] / prof_steps, 3) for k, v in prof.items()
              if isinstance(v, tuple) and k not in ("gemm", "gemm_wide", "ndb_fused")}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        c_ms, sample, threads = oracle_sample(spec, args)
        cpu = {"value": round(c_ms, 1), "unit": "ms", "cores": threads, "kind": "oracle", "sample": sample}

    line = {"metric": "Shampoo optimizer step ms", "value": round(ms, 3), "unit": "ms", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": False,
            "scaling": "strong", "vs_baseline": None,
            "dtype": "f32 (3 x fp16-split tensor products, fp32 accumulate)" if args.solver != "cn16" else
                     "f16 products, f32 accumulate",
            "data": "synthetic",
            "config": arm_config(args, spec, world), "state": ctx_info,
            "roofline": roofline, "inverse_root": inverse_root, "stage_ms": stages,
            "gpu_launches": launches, "clocks": clock_info, "e2e": e2e, "cpu_baseline": cpu}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
