"""QSA hot-path benchmark on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One "step" is one pass of the whole hot path (RoPE, indexer, top-k select,
sparse attention; for decode also the cache append and the split-KV combine)
over one batch of synthetic input resident in HBM, through the C ABI.  The
default workload is the 1M-token prefill; decode 64 x 256K and the 128K
prefill are measured in the same run as secondary lines.  With --gpus N (one
process per GPU under torchrun) every rank runs its own independent sequence
(weak scaling, no collective: sequences are independent problems).

--impl reference times the CPU oracle (the deliberately slow fp64 definition)
on a bounded sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import qsa_inputs as Q  # noqa: E402

L2_BYTES = 126 * (1 << 20)
DECODE_CALLS = 32          # decode tokens per sequence in one bench step (the workload's 32 steps)


def peaks():
    try:
        m = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"], bf16_sus=m["bf16_tflops_sustained"], src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=subprocess.PIPE,
                                      stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.p is not None:
            self.p.terminate()
            try:
                out, _ = self.p.communicate(timeout=5)
            except Exception:
                self.p.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- distributed
def dist_setup(n_gpus: int, backend: str | None = None):
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the
    launcher).  NCCL on GPUs; gloo when there is no GPU (the host-side tests)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if world > 1:
        import datetime
        if cuda:
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend or ("nccl" if cuda else "gloo"),
                                             timeout=datetime.timedelta(seconds=600))
    elif cuda:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: every rank's number, reduced with MAX."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Weak scaling: every rank draws its own independent sequences."""
    return seed + 1000 * rank


# ------------------------------------------------------------ prefill workload
def prefill_flops(T: int, sel_cnt: np.ndarray | None):
    """Algorithmic tensor FLOPs: indexer 1024 * T(T+1)/2 (4 heads x 128 x 2 per
    causal token pair); attention 4 * 24 * 256 * sum_t |J(t)| (QK^T and PV)."""
    idx = 1024.0 * T * (T + 1) / 2
    if sel_cnt is None:
        keys = min(T, 2048) * T
    else:
        # |J(t)| = 4 * cnt - (tokens of the own block after t)
        keys = float(4 * sel_cnt.astype(np.int64).sum() * 4) - 6.0 * len(sel_cnt)
    attn = 4.0 * 24 * 256 * keys
    return idx, attn


def run_prefill(T: int, budget: int, steps: int, warmup: int, rank: int, world: int, seed: int, want_e2e=True,
                aggregation: int = 0, idx_rope: int = 0):
    import block_sparse_long_qsa_b200 as qsa
    P = Q.PrefillProblem(T=T, seed=rank_seed(seed, rank), n_plant=8, dist="zipf" if T >= 131072 else "uniform")
    d = P.device()
    torch.cuda.synchronize()
    p = qsa.params(budget, aggregation=aggregation, idx_rope=idx_rope)
    mn, pref = qsa.qsa_prefill_workspace_size(p, T)
    ws = qsa.workspace(pref)
    nqb = P.nqb
    out = torch.empty((T, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((nqb, budget), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nqb,), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        qsa.qsa_prefill(p, T, 0, d["q"], d["k"], d["v"], d["q_idx"], d["w"], d["k_idx"], out, None, sel, cnt, None,
                        ws, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if qsa.qsa_check_device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk, qsa.trace(capacity=64 * steps + 64) as tr:
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world)
    if qsa.qsa_check_device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")
    cnt_h = cnt.cpu().numpy()
    fl_idx, fl_attn = prefill_flops(T, cnt_h)
    if aggregation == 1:
        fl_idx /= 4          # one compressed key per block: a quarter of the dot products
    kern = tr.by_kernel()
    launches = sum(c for c, _ in kern.values())
    res = dict(ms=ms_max, tokens=T * steps * world, kern=kern, launches=launches, clocks=clk.summary(),
               flops_idx=fl_idx, flops_attn=fl_attn, steps=steps,
               # K and V rows the attention gathers per step: 4 keys x 2 KV heads x 2 x 512 B per selected block
               gather_bytes=float(cnt_h.astype(np.int64).sum()) * 8192.0)

    if want_e2e:
        # end to end through the public call with host buffers: pinned inputs
        # copied in, the attention output copied back, every step
        # (pipelined: step i+1's inputs are copied in on one stream and step
        # i-1's output copied out on another while step i computes; device
        # input and output buffers are double-buffered)
        names = ["q", "k", "v", "q_idx", "w", "k_idx"]
        host = {k: torch.empty(d[k].shape, dtype=d[k].dtype, pin_memory=True) for k in names}
        for k in names:
            host[k].copy_(d[k])
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dins = [d, {k: torch.empty_like(d[k]) for k in names}]
        douts = [out, torch.empty_like(out)]
        torch.cuda.synchronize()
        bi = sum(host[k].numel() * host[k].element_size() for k in names)
        bo = out_h.numel() * out_h.element_size()
        # as many pipelined steps as the device-timed region (the first step's
        # input copy and the last step's output copy are not hidden)
        e_steps = max(2, steps)
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        in_ready = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n):
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(comp_done[b])      # step i-2 finished reading dins[b]
                    for k in names:
                        dins[b][k].copy_(host[k], non_blocking=True)
                    in_ready[b].record(s_in)
                stream.wait_event(in_ready[b])
                if i >= 2:
                    stream.wait_event(out_done[b])         # step i-2's output copied out of douts[b]
                x = dins[b]
                qsa.qsa_prefill(p, T, 0, x["q"], x["k"], x["v"], x["q_idx"], x["w"], x["k_idx"], douts[b], None,
                                sel, cnt, None, ws, stream)
                comp_done[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[b])
                    out_h.copy_(douts[b], non_blocking=True)
                    out_done[b].record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        stream.wait_event(e0)
        e2e_run(e_steps)
        e1.record(s_out)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        res["e2e"] = dict(value=T * e_steps * world / (ems / 1e3), unit="tokens/s", h2d_bytes_per_step=bi,
                          d2h_bytes_per_step=bo, steps=e_steps, pipelined=True)
        del host, out_h, dins, douts
    del d, ws, out, sel
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------- decode workload
def run_prefill_cached(T: int, L_old: int, budget: int, steps: int, warmup: int, rank: int, world: int, seed: int,
                       want_e2e=True):
    """Prefix-cached prefill: the first L_old tokens are in the caches, a step
    prefills the remaining T - L_old (qsa_prefill_cached); every step rewrites
    the same cache rows with the same values."""
    import block_sparse_long_qsa_b200 as qsa
    T_new = T - L_old
    P = Q.PrefillProblem(T=T, seed=rank_seed(seed, rank), n_plant=8, dist="zipf" if T >= 131072 else "uniform")
    d = P.device()
    # caches: synthetic keys stand in for rotated ones (timing only)
    kc, vc, ic = d["k"].clone(), d["v"].clone(), d["k_idx"].clone()
    t0 = 4 * (L_old // 4)
    qprev, wprev = d["q_idx"][t0:L_old].clone(), d["w"][t0:L_old].clone()
    new = {k: d[k][L_old:].clone() for k in ("q", "k", "v", "q_idx", "w", "k_idx")}
    del d
    torch.cuda.synchronize()
    p = qsa.params(budget)
    _, pref = qsa.qsa_prefill_cached_workspace_size(p, L_old, T_new)
    ws = qsa.workspace(pref)
    nq = (T + 3) // 4 - L_old // 4
    out = torch.empty((T_new, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((nq, budget), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nq,), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(x=None, o=None):
        x = x or new
        qsa.qsa_prefill_cached(p, L_old, T_new, kc, vc, ic, qprev if t0 < L_old else None,
                               wprev if t0 < L_old else None, x["q"], x["k"], x["v"], x["q_idx"], x["w"], x["k_idx"],
                               out if o is None else o, None, sel, cnt, ws, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if qsa.qsa_check_device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk, qsa.trace(capacity=64 * steps + 64) as tr:
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world)
    if qsa.qsa_check_device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")
    cnt_h = cnt.cpu().numpy().astype(np.int64)
    # indexer: every token of the new query blocks against all earlier keys;
    # attention: the new tokens over their selected keys
    first = 4 * (L_old // 4)
    fl_idx = 1024.0 * (T * (T + 1) / 2 - first * (first + 1) / 2)
    keys = float(16 * cnt_h.sum()) - 6.0 * len(cnt_h)
    fl_attn = 4.0 * 24 * 256 * keys * T_new / (T - first)
    kern = tr.by_kernel()
    res = dict(ms=ms_max, tokens=T_new * steps * world, kern=kern, launches=sum(c for c, _ in kern.values()),
               clocks=clk.summary(), flops_idx=fl_idx, flops_attn=fl_attn, steps=steps)
    if want_e2e:
        # new tokens' inputs copied in from pinned host memory and the output
        # copied back every step (serial; the cached prefix stays resident)
        names = ["q", "k", "v", "q_idx", "w", "k_idx"]
        host = {k: torch.empty(new[k].shape, dtype=new[k].dtype, pin_memory=True) for k in names}
        for k in names:
            host[k].copy_(new[k])
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dx = {k: torch.empty_like(new[k]) for k in names}
        bi = sum(host[k].numel() * host[k].element_size() for k in names)
        bo = out_h.numel() * out_h.element_size()
        e_steps = max(2, min(steps, 4))
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            for k in names:
                dx[k].copy_(host[k], non_blocking=True)
            step(dx)
            out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        res["e2e"] = dict(value=T_new * e_steps * world / (ems / 1e3), unit="tokens/s", h2d_bytes_per_step=bi,
                          d2h_bytes_per_step=bo, steps=e_steps, pipelined=False)
    del ws, kc, vc, ic, new
    torch.cuda.empty_cache()
    return res


def run_decode(B: int, L: int, budget: int, steps: int, warmup: int, rank: int, world: int, seed: int,
               want_e2e=True, aggregation: int = 0, spec: int = 0, verify_m: int = 0):
    import block_sparse_long_qsa_b200 as qsa
    # one bench step = DECODE_CALLS consecutive decode tokens per sequence; with
    # spec = n they form rounds of n draft steps: a full decode step, whose
    # selection the next n - 1 steps reuse (qsa_decode_reuse)
    # with verify_m = m every call is one qsa_verify of m new tokens per
    # sequence (all accepted: the next call starts m positions later)
    per_call = verify_m if verify_m else 1
    e_steps = max(1, min(steps, 3)) if want_e2e else 0
    n_calls = (warmup + steps + e_steps) * DECODE_CALLS
    D = Q.DecodeProblem(B=B, L=L, steps=n_calls * per_call, seed=rank_seed(seed, rank), n_plant=8)
    max_len = L + n_calls * per_call + 4
    kc = torch.empty((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.empty_like(kc)
    ic = torch.empty((B, max_len, 128), dtype=torch.uint16, device="cuda")
    D.fill_device_caches(kc, vc, ic)
    ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
    p = qsa.params(budget, aggregation=aggregation)
    kbar = None
    if aggregation == 1:
        # compressed-key cache of the cached prompt, kept up to date by each call
        kbar = torch.zeros((B, (max_len + 3) // 4, 128), dtype=torch.uint16, device="cuda")
        for b in range(B):
            qsa.qsa_mean_pool_keys(p, L, ic[b], kbar[b])
    ws = qsa.workspace(qsa.qsa_verify_workspace_size(p, B, verify_m, max_len) if verify_m else
                       qsa.qsa_decode_workspace_size(p, B, max_len))
    out = torch.empty((B, per_call, 24, 256) if verify_m else (B, 24, 256), dtype=torch.uint16, device="cuda")
    sel_round = torch.empty((B, budget), dtype=torch.int32, device="cuda") if spec > 1 else None
    # decode-token inputs of every call, generated once per sequence and kept resident: [call][B][...]
    names = ["q", "k", "v", "q_idx", "k_idx", "w"]
    per_seq = [D.tokens(b) for b in range(B)]
    allin = {}
    for k in names:
        arr = np.stack([getattr(per_seq[b], k)(L, L + n_calls * per_call) for b in range(B)], axis=1)
        if verify_m:   # [call][B][m][...]
            arr = arr.reshape(n_calls, per_call, *arr.shape[1:]).swapaxes(1, 2)
        allin[k] = torch.from_numpy(np.ascontiguousarray(arr)).cuda()
    step_in = [{k: allin[k][s] for k in names} for s in range(n_calls)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    pos = [L]

    def call(x):
        if verify_m:
            qsa.qsa_verify(p, B, verify_m, max_len, [pos[0]] * B, kc, vc, ic, ring, wring, x["q"], x["k"], x["v"],
                           x["q_idx"], x["k_idx"], x["w"], out, ws=ws, stream=stream)
            pos[0] += verify_m
            return
        if spec > 1 and (pos[0] - L) % spec != 0:
            qsa.qsa_decode_reuse(p, B, max_len, [pos[0]] * B, kc, vc, ic, kbar, ring, wring, x["q"], x["k"], x["v"],
                                 x["q_idx"], x["k_idx"], x["w"], sel_round, None, out, ws=ws, stream=stream)
        elif kbar is None:
            qsa.qsa_decode(p, B, max_len, [pos[0]] * B, kc, vc, ic, ring, wring, x["q"], x["k"], x["v"], x["q_idx"],
                           x["k_idx"], x["w"], out, sel_out=sel_round, ws=ws, stream=stream)
        else:
            qsa.qsa_decode_mean_pool(p, B, max_len, [pos[0]] * B, kc, vc, ic, kbar, ring, wring, x["q"], x["k"],
                                     x["v"], x["q_idx"], x["k_idx"], x["w"], out, sel_out=sel_round, ws=ws,
                                     stream=stream)
        pos[0] += 1

    si = 0

    def step():
        nonlocal si
        for _ in range(DECODE_CALLS):
            call(step_in[si]); si += 1

    # the clock sampler starts before the warm-up so that its start-up does not
    # overlap the (short) timed region
    clk = ClockSampler(torch.cuda.current_device()).__enter__()
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if qsa.qsa_check_device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    L_first = pos[0]
    with qsa.trace(capacity=16 * steps * DECODE_CALLS + 16) as tr:
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    clk.__exit__(None, None, None)
    barrier(world)
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world)
    if qsa.qsa_check_device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")
    kern = tr.by_kernel()
    # algorithmic bytes per decode call: every cached indexer key (256 B) read
    # once, the gathered K and V rows of the selected blocks, the appended token
    # and the inputs / outputs
    n_timed = steps * DECODE_CALLS
    # keys: every cached indexer key read once per call (the algorithmic
    # figure, also for a verify whose query blocks each read them)
    keys = B * (L_first + n_timed * per_call / 2 + 1)
    if aggregation == 1:
        keys /= 4            # one 256-byte compressed key per block
    gathered = per_call * B * min(budget, L_first // 4 + 1) * 4 * 2 * 2 * 256 * 2
    io = per_call * B * (24 * 256 * 2 * 2 + 2 * 2 * 256 * 2 + 128 * 2 * 2)
    # the indexer keys are read only by the calls that select
    select_share = 1.0 / spec if spec > 1 else 1.0
    bytes_call = keys * 256 * select_share + gathered + io
    res = dict(ms=ms_max, tokens=B * n_timed * per_call * world, kern=kern,
               launches=sum(c for c, _ in kern.values()), clocks=clk.summary(), bytes_step=bytes_call * DECODE_CALLS,
               bytes_indexer=keys * 256, steps=steps, calls=n_timed)
    if want_e2e:
        # every call: that call's inputs copied in from pinned host memory, the
        # output copied back
        hosts = {k: torch.empty(allin[k].shape, dtype=allin[k].dtype, pin_memory=True) for k in names}
        for k in names:
            hosts[k].copy_(allin[k])
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        bi = sum(step_in[0][k].numel() * step_in[0][k].element_size() for k in names) * DECODE_CALLS
        bo = out_h.numel() * out_h.element_size() * DECODE_CALLS
        xdev = {k: torch.empty_like(step_in[0][k]) for k in names}

        def e2e_step():
            nonlocal si
            for _ in range(DECODE_CALLS):
                for k in names:
                    xdev[k].copy_(hosts[k][si], non_blocking=True)
                call(xdev)
                si += 1
                out_h.copy_(out, non_blocking=True)

        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        res["e2e"] = dict(value=B * DECODE_CALLS * per_call * e_steps * world / (ems / 1e3), unit="tokens/s",
                          h2d_bytes_per_step=bi, d2h_bytes_per_step=bo, steps=e_steps)
        del hosts, out_h
    del kc, vc, ic, ws, step_in, allin, kbar, sel_round
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------ CPU baselines
_KIDX_CACHE: dict = {}


def cpu_sample(wl: dict, target_s: float = 12.0, stratified: int = 0):
    """The oracle on a bounded sample of the workload sized to ~target_s of
    CPU time: a calibration run, then one run scaled to the target.  With
    stratified = n (prefill only) the sample is instead the n stratified query
    blocks the parity checks use."""
    if stratified and wl["kind"] == "prefill":
        return cpu_prefill_sample(wl["T"], 512, stratified, aggregation=wl.get("aggregation", 0), stratified=True,
                                  idx_rope=wl.get("idx_rope", 0))
    if wl["kind"] in ("prefill", "prefill_cached"):
        qb_lo = wl.get("L_old", 0) // 4
        agg = wl.get("aggregation", 0)
        n = max(4, cores_used())
        rope = wl.get("idx_rope", 0)
        v, info = cpu_prefill_sample(wl["T"], 512, n, qb_lo=qb_lo, aggregation=agg, idx_rope=rope)
        if info["elapsed"] < target_s / 3:
            n2 = int(min((wl["T"] + 3) // 4 - qb_lo, max(n + 1, n * target_s / max(info["elapsed"], 1e-3))))
            v, info = cpu_prefill_sample(wl["T"], 512, n2, qb_lo=qb_lo, aggregation=agg, idx_rope=rope)
    else:
        n = 2
        agg = wl.get("aggregation", 0)
        spec = wl.get("spec", 0)
        if wl.get("verify_m"):
            return cpu_verify_sample(wl["B"], wl["L"], 512, wl["verify_m"], target_s)
        v, info = cpu_decode_sample(wl["B"], wl["L"], 512, n, aggregation=agg, spec=spec)
        if info["elapsed"] < target_s / 3:
            n2 = int(min(wl["B"], max(n + 1, n * target_s / max(info["elapsed"], 1e-3))))
            v, info = cpu_decode_sample(wl["B"], wl["L"], 512, n2, aggregation=agg, spec=spec)
    return v, info


def _oracle_work(qbs: np.ndarray, T: int, budget: int) -> np.ndarray:
    """Multiply-adds the oracle spends on query block qb: scores (16 token
    pairs x 4 heads x 128 dims per causal key block) plus attention (4 tokens
    x 24 heads x 2 x 256 per attended key)."""
    qbs = np.asarray(qbs, dtype=np.float64)
    n_tok = np.minimum(4.0, T - 4.0 * qbs)
    keys = np.minimum(4.0 * (qbs + 1), 4.0 * budget)
    return 16 * 512 * (qbs + 1) + n_tok * 24 * 512 * keys


def cpu_prefill_sample(T: int, budget: int, n_blocks: int, seed: int = 0, qb_lo: int = 0, aggregation: int = 0,
                       stratified: bool = False, idx_rope: int = 0):
    """The oracle on a sample of query blocks of the T-token prefill (evenly
    spaced in [qb_lo, nqb), or the stratified sample of the parity checks),
    all host cores.  Returns tokens/s of the oracle extrapolated to the whole
    workload by the sample's share of the oracle's multiply-adds, and a
    description."""
    import oracle
    O = oracle.Oracle(oracle.params(budget=budget, aggregation=aggregation, idx_rope=idx_rope))
    P = Q.PrefillProblem(T=T, seed=seed, n_plant=8, dist="zipf" if T >= 131072 else "uniform")
    nqb = P.nqb
    if stratified:
        qbs = Q.stratified_query_blocks(nqb, n=n_blocks, budget=budget, seed=T)
        qbs = qbs[qbs >= qb_lo]
    else:
        qbs = np.unique(np.linspace(qb_lo, nqb - 1, n_blocks).astype(np.int64))
    key = (T, seed)
    if key not in _KIDX_CACHE:
        _KIDX_CACHE.clear()
        _KIDX_CACHE[key] = P.k_idx(0, T)
    k_idx = _KIDX_CACHE[key]
    q_idx = np.zeros((T, 4, 128), np.uint16)
    w = np.zeros((T, 4), np.uint16)
    for qb in qbs:
        t0, t1 = qb * 4, min(qb * 4 + 4, T)
        q_idx[t0:t1] = P.q_idx(t0, t1)
        w[t0:t1] = P.w(t0, t1)
    kfull = np.zeros((T, 128), np.uint16)
    kfull[:k_idx.shape[0]] = k_idx
    # scores + selection (timed)
    t_a = time.time()
    sel, cnt = O.select_blocks_list(T, q_idx, w, kfull, qbs)
    t_score = time.time() - t_a
    # attention inputs for the selected blocks (untimed)
    q = np.zeros((T, 24, 256), np.uint16)
    k = np.zeros((T, 2, 256), np.uint16)
    v = np.zeros((T, 2, 256), np.uint16)
    for i, qb in enumerate(qbs):
        t0, t1 = qb * 4, min(qb * 4 + 4, T)
        q[t0:t1] = P.q(t0, t1)
        for b in sel[i][:cnt[i]]:
            a0, a1 = b * 4, min(b * 4 + 4, T)
            k[a0:a1] = P.k(a0, a1)
            v[a0:a1] = P.v(a0, a1)
    t_b = time.time()
    O.attend_blocks(T, q, k, v, qbs, sel, cnt)
    t_attn = time.time() - t_b
    elapsed = t_score + t_attn
    all_q = np.arange(qb_lo, nqb)
    share = _oracle_work(qbs, T, budget).sum() / _oracle_work(all_q, T, budget).sum()
    tokens = T - 4 * qb_lo
    span = "" if qb_lo == 0 else f" from query block {qb_lo} on"
    kind = "stratified (first, last, around the budget boundary, evenly spaced)" if stratified else "evenly spaced"
    return tokens * share / elapsed, dict(
        sample=f"{len(qbs)} {kind} query blocks{span} of the {T}-token prefill (scores + selection + attention), "
               f"{elapsed:.1f} s, extrapolated by their {100 * share:.3f} % share of the oracle's multiply-adds",
        elapsed=elapsed)


def cpu_decode_sample(B: int, L: int, budget: int, n_seq: int, seed: int = 0, aggregation: int = 0,
                      spec: int = 0):
    import oracle
    O = oracle.Oracle(oracle.params(budget=budget, aggregation=aggregation))
    D = Q.DecodeProblem(B=B, L=L, steps=1, seed=seed, n_plant=8)
    elapsed = 0.0
    for b in range(n_seq):
        P = D.tokens(b)
        kid = D.cache_kidx(b)
        x = {k: getattr(P, k)(L, L + 1)[0] for k in ("q", "k", "v", "q_idx", "w")}
        kidx_new = P.k_idx(L, L + 1)[0]
        # selection first (timed) to know which cache rows attention needs
        t0 = time.time()
        S = O.block_scores(L // 4, x["q_idx"][None], x["w"][None],
                           np.concatenate([kid, kidx_new[None]]))
        sel, cnt = O.select(L // 4, S)
        t_sel = time.time() - t0
        kc = np.zeros((L, 2, 256), np.uint16)
        vc = np.zeros((L, 2, 256), np.uint16)
        for blk in sel[:cnt]:
            a0, a1 = blk * 4, min(blk * 4 + 4, L)
            if a1 > a0:
                kc[a0:a1] = D.cache_k(b, a0, a1)
                vc[a0:a1] = D.cache_v(b, a0, a1)
        # attention on that selection (timed); with spec = n also the n - 1
        # draft tokens of the round that reuse it
        t1 = time.time()
        # no block-mates before token L: the workload's L is a multiple of 4
        ring_q, ring_w = P.q_idx(4 * (L // 4), L), P.w(4 * (L // 4), L)
        O.decode(L, kc, vc, kid, ring_q, ring_w, x["q"], x["k"], x["v"], x["q_idx"], kidx_new, x["w"],
                 sel_in=sel, cnt_in=cnt)
        for _ in range(max(spec, 1) - 1):
            O.decode_reuse(L, kc, vc, kid, ring_q, ring_w, x["q"], x["k"], x["v"], x["q_idx"], kidx_new, x["w"],
                           sel_in=sel, cnt_in=cnt)
        elapsed += t_sel + (time.time() - t1)
    per = max(spec, 1)
    what = ("one decode token each" if per == 1 else
            f"a round of {per} draft tokens each (one selection, {per - 1} reusing it; all at position {L})")
    return n_seq * per / elapsed, dict(sample=f"{n_seq} of {B} sequences, {what} at {L} cached tokens "
                                              f"(scores + selection + attention), {elapsed:.1f} s", elapsed=elapsed)


def cpu_verify_sample(B: int, L: int, budget: int, m: int, target_s: float = 12.0, seed: int = 0):
    """The oracle on sampled sequences of a verify call: each query block the
    m new tokens touch is scored over the cached keys and selected, then each
    new token attends its block's selection (the cached K / V rows the
    selection needs are materialised untimed; rows of earlier new tokens are
    left zero -- the work per token is the same)."""
    import oracle
    O = oracle.Oracle(oracle.params(budget=budget))
    D = Q.DecodeProblem(B=B, L=L, steps=m, seed=seed, n_plant=8)
    elapsed, n_seq = 0.0, 0
    while n_seq < B and (elapsed < target_s / 2 or n_seq < 1):
        b = n_seq
        P = D.tokens(b)
        kid = np.concatenate([D.cache_kidx(b), P.k_idx(L, L + m)])
        x = {k: getattr(P, k)(L, L + m) for k in ("q", "k", "v", "q_idx", "w")}
        for qb in sorted({(L + i) // 4 for i in range(m)}):
            t0, t1 = max(4 * qb, L), min(4 * qb + 4, L + m)
            ta = time.time()
            S = O.block_scores(qb, x["q_idx"][t0 - L:t1 - L], x["w"][t0 - L:t1 - L], kid[:t1])
            sel, cnt = O.select(qb, S)
            elapsed += time.time() - ta
            kc = np.zeros((t1, 2, 256), np.uint16)
            vc = np.zeros((t1, 2, 256), np.uint16)
            for blk in sel[:cnt]:
                a0, a1 = blk * 4, min(blk * 4 + 4, L)
                if a1 > a0:
                    kc[a0:a1] = D.cache_k(b, a0, a1)
                    vc[a0:a1] = D.cache_v(b, a0, a1)
            for t in range(t0, t1):
                i = t - L
                tb = time.time()
                # block-mates 4 qb .. t - 1: cached tokens before L, new tokens from L on
                c1 = max(4 * qb, min(L, t))
                mates_q = np.concatenate([P.q_idx(4 * qb, c1), x["q_idx"][max(4 * qb, L) - L:i]])
                mates_w = np.concatenate([P.w(4 * qb, c1), x["w"][max(4 * qb, L) - L:i]])
                O.decode(t, kc[:t], vc[:t], kid[:t], mates_q, mates_w, x["q"][i], x["k"][i], x["v"][i],
                         x["q_idx"][i], kid[t], x["w"][i], sel_in=sel, cnt_in=cnt)
                elapsed += time.time() - tb
        n_seq += 1
    return n_seq * m / elapsed, dict(sample=f"{n_seq} of {B} sequences, {m} verify tokens each at {L} cached tokens "
                                            f"(scores + selection per touched block, attention per token), "
                                            f"{elapsed:.1f} s", elapsed=elapsed)


def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


# ------------------------------------------------------------------- main
WORKLOADS = {
    "prefill_1m": dict(kind="prefill", T=1 << 20),
    "prefill_128k": dict(kind="prefill", T=131072),
    "prefill_32k": dict(kind="prefill", T=32768),
    "decode_64x256k": dict(kind="decode", B=64, L=262144),
    # 90 % of a 1M-token prompt already cached (L_old % 4 = 2: the first new
    # query block starts mid-block)
    "prefill_1m_cached90": dict(kind="prefill_cached", T=1 << 20, L_old=943718),
    # the pages' mean-pooled indexer (one compressed key per 4-token block)
    "prefill_1m_meanpool": dict(kind="prefill", T=1 << 20, aggregation=1),
    # the same with the indexer's RoPE: queries rotated at their token, each
    # compressed key at its block's first token
    "prefill_1m_meanpool_rope": dict(kind="prefill", T=1 << 20, aggregation=1, idx_rope=1),
    "decode_64x256k_meanpool": dict(kind="decode", B=64, L=262144, aggregation=1),
    # speculative rounds of 4 draft tokens: one selection, reused by the next 3
    "decode_64x256k_spec4": dict(kind="decode", B=64, L=262144, spec=4),
    # target-model verify of 5 draft tokens per sequence per call (all accepted)
    "verify_64x256k_m5": dict(kind="decode", B=64, L=262144, verify_m=5),
}


# DRAM bytes per launch of the dominant kernel (dram__bytes_read.sum +
# dram__bytes_write.sum) with the current kernels; None where no capture exists.
# prefill_1m: from a small-case capture of the indexer (the last 2,048 query
# blocks of the 1M-token problem: 522K units, 0.357 GB read, 2.09 GB written),
# the reads scaled to the mean launch of the 1M prefill by units (3.36M, an
# upper bound: key bands are read once per band) and the writes (the score
# slab and segment maxima, in proportion to the causal entries) 15.46 GB.
# The decode figures are averaged launches of one-pass captures.
NCU_TRAFFIC = {"prefill_1m": 0.357e9 * 3.36 / 0.522 + 15.46e9, "decode_64x256k": 4.2954e9 + 0.0093e9,
               "decode_64x256k_spec4": 4.2957e9 + 0.0085e9, "verify_64x256k_m5": 4.2982e9 + 0.0084e9}


def metric_name(wl: dict) -> str:
    if wl["kind"] == "prefill":
        mp = ", mean-pooled indexer" if wl.get("aggregation") == 1 else ""
        if wl.get("idx_rope"):
            mp += " with block-start RoPE"
        return f"QSA prefill tokens/s at {wl['T'] // 1024}K context{mp}"
    if wl["kind"] == "prefill_cached":
        return (f"QSA prefix-cached prefill new tokens/s at {wl['T'] // 1024}K context, "
                f"{round(100 * wl['L_old'] / wl['T'])}% cached")
    mp = ", mean-pooled indexer" if wl.get("aggregation") == 1 else ""
    if wl.get("spec"):
        mp += f", top-k reused across {wl['spec']}-step speculative rounds"
    if wl.get("verify_m"):
        return f"QSA verified tokens/s at 256K context, batch 64, {wl['verify_m']} tokens per sequence per call"
    return f"QSA decode tokens/s at 256K context, batch 64{mp}"


def line_for(name, res, n_gpus, steps, warmup, pk):
    wl = WORKLOADS[name]
    if wl["kind"] in ("prefill", "prefill_cached"):
        T = wl["T"]
        value = res["tokens"] / (res["ms"] / 1e3)
        idx_n, idx_ms = res["kern"].get("indexer", (1, float("nan")))
        # achieved = algorithmic indexer FLOPs per launch / mean launch time
        achieved = res["flops_idx"] * res["steps"] / idx_n / (idx_ms / idx_n / 1e3) / 1e12
        roof = dict(kernel="indexer", bound="tensor", achieved=achieved, peak=pk["bf16_sus"], unit="TFLOP/s",
                    frac=achieved / pk["bf16_sus"], traffic=NCU_TRAFFIC.get(name),
                    peak_src=f"{pk['src']} bf16 dense sustained")
        total_fl = res["flops_idx"] + res["flops_attn"]
        whole = dict(tflops=total_fl / (res["ms"] / res["steps"] / 1e3) / 1e12)
        if "gather_bytes" in res and "attention" in res["kern"]:
            # the attention against its own bound: gathered K / V bytes (L2 hits
            # included) per second against the HBM copy bandwidth
            att_s = res["kern"]["attention"][1] / res["steps"] / 1e3
            gbs = res["gather_bytes"] / att_s / 1e9
            whole["attention"] = dict(bound="hbm", gathered_gb_per_step=round(res["gather_bytes"] / 1e9, 2),
                                      achieved_gbs=round(gbs, 1), frac_of_hbm=round(gbs / pk["hbm"], 4),
                                      tflops=round(res["flops_attn"] / att_s / 1e12, 1))
        whole["frac_of_tensor_roofline"] = whole["tflops"] / pk["bf16_sus"]
        metric = metric_name(wl)
        cfg = dict(workload=name, T=T, batch=1, budget_blocks=512, heads="24q/2kv x 256, idx 4 x 128",
                   planted="8/query block, " + ("zipf(1.1) distance" if T >= 131072 else "uniform"),
                   l2="inputs larger than L2 (126 MB): no flush needed")
        if "L_old" in wl:
            cfg.update(cached_tokens=wl["L_old"], new_tokens=T - wl["L_old"])
    else:
        B, L = wl["B"], wl["L"]
        value = res["tokens"] / (res["ms"] / 1e3)
        n, t = res["kern"].get("decode_indexer", (1, float("nan")))
        achieved = res["bytes_indexer"] / (t / n / 1e3) / 1e9
        roof = dict(kernel="decode_indexer", bound="hbm", achieved=achieved, peak=pk["hbm"], unit="GB/s",
                    frac=achieved / pk["hbm"], traffic=NCU_TRAFFIC.get(name), peak_src=f"{pk['src']} HBM copy")
        whole = dict(gbs=res["bytes_step"] / (res["ms"] / res["steps"] / 1e3) / 1e9)
        whole["frac_of_hbm_roofline"] = whole["gbs"] / pk["hbm"]
        metric = metric_name(wl)
        cfg = dict(workload=name, batch=B, context=L, budget_blocks=512, planted="8 per sequence",
                   decode_tokens_per_step=DECODE_CALLS * (wl.get("verify_m") or 1),
                   speculative_round=wl.get("spec") or None, verify_tokens_per_call=wl.get("verify_m") or None,
                   l2=("1.07 GB of compressed indexer keys" if wl.get("aggregation") == 1 else
                       "4.3 GB of indexer keys") + " streamed per decode token (larger than L2)")
    return dict(metric=metric, value=value, unit="tokens/s", n_gpus=n_gpus, steps=steps, warmup=warmup,
                ms_per_step=res["ms"] / steps, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="bf16", data="synthetic", config=cfg, roofline=roof, step_roofline=whole,
                clocks=res["clocks"], gpu_launches=res["launches"], e2e=res.get("e2e"),
                kernels_ms={k: dict(launches=c, total_ms=round(tt, 3)) for k, (c, tt) in res["kern"].items()})


def ncu_case(spec: str):
    """A small case of the hot path for profiler captures (not a benchmark)."""
    import block_sparse_long_qsa_b200 as qsa
    torch.cuda.set_device(0)
    parts = spec.split(":")
    if parts[0] == "prefill":
        T = int(parts[1])
        P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist="uniform")
        d = P.device()
        for _ in range(2):
            r = qsa.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["w"], d["k_idx"], budget=512, want_lse=False)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(r["ws"]) == 0
    elif parts[0] == "indextail":
        # stage 1 alone over the last `rows` query blocks of a T-token problem
        # (keys larger than L2, a few GB on the device), three launches
        T, rows = int(parts[1]), int(parts[2])
        P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist="zipf")
        d = P.device()
        p = qsa.params(512)
        nqb = (T + 3) // 4
        ld = (nqb + 3) // 4 * 4
        S = torch.empty((rows, ld), dtype=torch.float32, device="cuda")
        ws = qsa.workspace(qsa.qsa_index_workspace_size(p, T))
        for _ in range(3):
            qsa.qsa_index_scores(p, T, d["q_idx"], d["w"], d["k_idx"], nqb - rows, nqb, S, ld, ws)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(ws) == 0
    elif parts[0] == "attntail":
        # the prefill of the last `rows` query blocks of a T-token problem over
        # the cached first T - 4 rows tokens (qsa_prefill_cached): the
        # attention gathers from a T-token cache larger than L2, a few GB on
        # the device; the full q is never generated (indexer keys unplanted)
        T, rows = int(parts[1]), int(parts[2])
        T_new = 4 * rows
        L_old = T - T_new
        P = Q.PrefillProblem(T=T, seed=0, n_plant=0, dist="zipf")
        kc, vc, ic = (P.device_rows(n, 0, T) for n in ("k", "v", "k_idx"))
        new = {n: P.device_rows(n, L_old, T) for n in ("q", "k", "v", "q_idx", "w", "k_idx")}
        p = qsa.params(512)
        _, pref = qsa.qsa_prefill_cached_workspace_size(p, L_old, T_new)
        ws = qsa.workspace(pref)
        out = torch.empty((T_new, 24, 256), dtype=torch.uint16, device="cuda")
        sel = torch.empty((rows, 512), dtype=torch.int32, device="cuda")
        cnt = torch.empty((rows,), dtype=torch.int32, device="cuda")
        for _ in range(2):
            qsa.qsa_prefill_cached(p, L_old, T_new, kc, vc, ic, None, None, new["q"], new["k"], new["v"],
                                   new["q_idx"], new["w"], new["k_idx"], out, None, sel, cnt, ws)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(ws) == 0
    elif parts[0] == "index":
        # stage 1 alone (qsa_index_scores, no segment maxima), four launches
        T = int(parts[1])
        P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist="uniform")
        d = P.device()
        p = qsa.params(512)
        nqb = (T + 3) // 4
        ld = (nqb + 3) // 4 * 4
        S = torch.empty((nqb, ld), dtype=torch.float32, device="cuda")
        ws = qsa.workspace(qsa.qsa_index_workspace_size(p, T))
        for _ in range(4):
            qsa.qsa_index_scores(p, T, d["q_idx"], d["w"], d["k_idx"], 0, nqb, S, ld, ws)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(ws) == 0
    else:
        B, L = int(parts[1]), int(parts[2])
        D = Q.DecodeProblem(B=B, L=L, steps=2, seed=0, n_plant=8)
        max_len = L + 8
        kc = torch.empty((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
        vc = torch.empty_like(kc)
        ic = torch.empty((B, max_len, 128), dtype=torch.uint16, device="cuda")
        D.fill_device_caches(kc, vc, ic)
        ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
        wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
        p = qsa.params(512)
        ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len))
        out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
        for s in range(2):
            x = {k: torch.from_numpy(v).cuda() for k, v in D.step_inputs(s).items()}
            kn = torch.zeros((B, 128), dtype=torch.uint16, device="cuda")
            qsa.qsa_decode(p, B, max_len, [L + s] * B, kc, vc, ic, ring, wring, x["q"], x["k"], x["v"], x["q_idx"],
                           kn, x["w"], out, ws=ws)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(ws) == 0
    print("ncu case done", spec)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_1m", choices=list(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ncu-case", default=None,
                    help="prefill:T, index:T, indextail:T:rows, attntail:T:rows or decode:B:L -- a few calls of a small case "
                         "(for ncu captures)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    if args.ncu_case:
        ncu_case(args.ncu_case)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        wl = WORKLOADS[args.workload]
        for _ in range(args.warmup):          # untimed, shorter samples of the same workload
            cpu_sample(wl, target_s=3.0)
        ts, descs, walls = [], [], []
        for _ in range(args.steps):
            v, info = cpu_sample(wl)
            ts.append(v)
            descs.append(info["sample"])
            walls.append(info["elapsed"] * 1e3)
        value = statistics.median(ts)
        cb = dict(value=value, unit="tokens/s", cores=cores_used(), kind="oracle", sample=descs[0])
        metric = metric_name(wl)
        print(json.dumps(dict(impl="reference", metric=metric, value=value, unit="tokens/s", n_gpus=args.gpus,
                              steps=args.steps, warmup=args.warmup,
                              ms_per_step=statistics.median(walls),   # one sampled step, not the whole workload
                              higher_is_better=True,
                              scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                              config=dict(workload=args.workload), cpu_baseline=cb,
                              e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))),
              flush=True)
        return

    rank, world, local = dist_setup(args.gpus)
    import block_sparse_long_qsa_b200 as qsa
    qsa.load()
    pk = peaks()
    wl = WORKLOADS[args.workload]
    if wl["kind"] == "prefill":
        res = run_prefill(wl["T"], 512, args.steps, args.warmup, rank, world, seed=0, want_e2e=not args.no_e2e,
                          aggregation=wl.get("aggregation", 0), idx_rope=wl.get("idx_rope", 0))
    elif wl["kind"] == "prefill_cached":
        res = run_prefill_cached(wl["T"], wl["L_old"], 512, args.steps, args.warmup, rank, world, seed=0,
                                 want_e2e=not args.no_e2e)
    else:
        res = run_decode(wl["B"], wl["L"], 512, args.steps, args.warmup, rank, world, seed=0,
                         want_e2e=not args.no_e2e, aggregation=wl.get("aggregation", 0), spec=wl.get("spec", 0),
                         verify_m=wl.get("verify_m", 0))
    line = line_for(args.workload, res, world, args.steps, args.warmup, pk)

    if rank == 0 and world == 1 and not args.no_cpu:
        # 256 stratified query blocks at 1M (about half a minute on 16 cores)
        v, info = cpu_sample(wl, stratified=256 if wl.get("T", 0) >= 1 << 20 else 0)
        line["cpu_baseline"] = dict(value=v, unit="tokens/s", cores=cores_used(), kind="oracle",
                                    sample=info["sample"])

    if not args.no_secondary:
        # the other workloads, compact (the line's end is what a log tail
        # keeps, so the plain decode and the 128K / 32K prefill come last)
        sec = {}
        for name in ("prefill_1m_cached90", "prefill_1m_meanpool", "prefill_1m_meanpool_rope",
                     "decode_64x256k_meanpool", "decode_64x256k_spec4",
                     "verify_64x256k_m5", "prefill_32k", "prefill_128k", "decode_64x256k"):
            if name == args.workload:
                continue
            w2 = WORKLOADS[name]
            if w2["kind"] == "prefill":
                r2 = run_prefill(w2["T"], 512, args.steps, args.warmup, rank, world, seed=0, want_e2e=False,
                                 aggregation=w2.get("aggregation", 0), idx_rope=w2.get("idx_rope", 0))
            elif w2["kind"] == "prefill_cached":
                r2 = run_prefill_cached(w2["T"], w2["L_old"], 512, args.steps, args.warmup, rank, world, seed=0,
                                        want_e2e=False)
            else:
                r2 = run_decode(w2["B"], w2["L"], 512, args.steps, args.warmup, rank, world, seed=0,
                                want_e2e=False, aggregation=w2.get("aggregation", 0), spec=w2.get("spec", 0),
                                verify_m=w2.get("verify_m", 0))
            l2 = line_for(name, r2, world, args.steps, args.warmup, pk)
            sr = l2["step_roofline"]
            sec[name] = dict(metric=l2["metric"], value=round(l2["value"], 1), ms_per_step=round(l2["ms_per_step"], 3),
                             kernel=l2["roofline"]["kernel"], kernel_frac=round(l2["roofline"]["frac"], 4),
                             step_frac=round(sr.get("frac_of_tensor_roofline", sr.get("frac_of_hbm_roofline")), 4))
            km = l2["kernels_ms"]
            for kname in ("attention", "decode_attention"):
                if kname in km:   # the attention's share of the step
                    sec[name][kname + "_ms_per_step"] = round(km[kname]["total_ms"] / args.steps, 3)
        line["secondary"] = sec

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
