#!/usr/bin/env python
"""Benchmark of the Llama-3-8B-shaped decoder forward pass on B200.

One step = one full-model prefill (32 layers, embedding, final norm, LM head,
greedy argmax) of B=1 sequence of 2048 seeded token ids, with N(0, 0.02)
seeded weights. The line's ``value`` is prefill tokens/s over all GPUs
(replicas: each rank runs its own model, no data-path collective). The same
run measures the batch-32 KV-cache decode workload (context 4096 filled with
N(0,1) K/V entries, 128 greedy steps at positions 4096..4223) under
``decode``.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --kernel attention_prefill|attention_decode|linear [shape flags]
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = 'tokens/s: 8B-shape prefill & batch-32 decode; % tensor/HBM roofline'
PREFILL_B, PREFILL_S = 1, 2048
PREFILL_B8 = 8
LONG_S, LONG_CHUNK = 32768, 4096       # long-context leg: one layer, chunked prefill
DECODE_B, DECODE_CTX, DECODE_STEPS = 32, 4096, 128


def _peaks():
    try:
        with open(os.path.join(ROOT, 'MEASURED_PEAKS.json')) as f:
            p = json.load(f)
        return p['hbm_gbs'], p['bf16_tflops'], p['bf16_tflops_sustained'], 'measured'
    except Exception:
        return 6650.0, 1590.0, 1400.0, 'fallback'


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling every 200 ms during a timed region (one background
    process, started before the region and stopped after it)."""
    FIELDS = ('index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,'
              'clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,'
              'clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap')

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(['nvidia-smi', '-i', str(self.idx), f'--query-gpu={self.FIELDS}',
                                          '--format=csv,noheader,nounits', '-lms', '200'],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)   # first sample before the region starts
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for ln in (out or '').strip().splitlines():
            self.rows.append([c.strip() for c in ln.split(',')])

    def summary(self):
        rows = [r for r in self.rows if len(r) >= 9]
        if not rows:
            return {'sm_mhz': None, 'sm_max_mhz': None, 'reasons': ['nvidia-smi unavailable'], 'samples': 0}
        sm = [float(r[1]) for r in rows if r[1].replace('.', '').isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace('.', '').isdigit()]
        names = ['hw_slowdown', 'hw_thermal_slowdown', 'sw_thermal_slowdown', 'sw_power_cap']
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == 'active'})
        return {'sm_mhz': statistics.median(sm) if sm else None, 'sm_max_mhz': max(mx) if mx else None,
                'reasons': reasons, 'samples': len(rows)}


# ------------------------------------------------------------ distributed
def _dist():
    ws = int(os.environ.get('WORLD_SIZE', '1'))
    rank = int(os.environ.get('RANK', '0'))
    local = int(os.environ.get('LOCAL_RANK', '0'))
    return ws, rank, local


def _max_over_ranks(x: float, ws: int) -> float:
    """Largest per-rank value (the replicas' step time is the slowest rank's)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = 'cpu' if dist.get_backend() == 'gloo' else 'cuda'
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, local_ms: float, ws: int):
    """Whole-job throughput of ws replicas that each process units_per_rank
    units in local_ms: (units/s over all ranks, the max-over-ranks ms)."""
    ms = _max_over_ranks(local_ms, ws)
    return ws * units_per_rank / (ms / 1e3), ms


def _barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------- CPU oracle sample
def oracle_threads() -> int:
    """Threads the oracle's numpy BLAS runs with (all host cores unless limited)."""
    try:
        from threadpoolctl import threadpool_info
        n = [p['num_threads'] for p in threadpool_info() if p.get('user_api') == 'blas']
        return max(n) if n else 1
    except Exception:  # pragma: no cover - threadpoolctl missing
        return os.cpu_count() or 1


class OracleSample:
    """The float32 CPU oracle, as it stands, on bounded samples of the 8B
    workloads. Weights of layer 0 and the output matrix are generated once,
    outside every timed region. Samples:

    * layer(S): one of the 32 decoder layers over S prompt tokens;
    * head(): embedding of the prompt, final norm and LM head of the last row;
    * decode_layer(ctx): one layer of one decode step (B = 1) over a cache of
      ctx positions of N(0,1) K/V entries.

    Full-model figures are derived from the timed samples as
    tokens / (32 x layer time + head time); every sample that enters one was
    timed in the same run."""

    def __init__(self):
        import numpy as np
        from oracle import Oracle, Params, SequenceCache
        import seeded_inputs as si
        self.np, self.si = np, si
        self.p = Params(4096, 32, 32, 8, 128256, 14336)

        class W(dict):
            def __missing__(self, name):
                if name.endswith('norm.weight'):
                    v = np.ones(4096, np.float32)
                else:
                    shape = si.weight_shape(name, 4096, 32, 8, 14336, 128256)
                    v = si.bf16_bits_to_f32(si.weight(0, name, shape, 32, 0.02, 'bf16'))
                self[name] = v
                return v

        self.w = W()
        for name in ['tok_embeddings.weight', 'output.weight', 'norm.weight'] + \
                [f'layers.0.{k}.weight' for k in si.LAYER_KEYS]:
            self.w[name]
        self.orc = Oracle(self.p, self.w, dtype=np.float32)
        self.SequenceCache = SequenceCache
        self._x = {}
        self._cache = None

    def _hidden(self, S):
        if S not in self._x:
            si = self.si
            self._x[S] = si.bf16_bits_to_f32(si.normal(2, si.STREAM_HIDDEN, S * 4096, 1.0)).reshape(S, 4096)
        return self._x[S]

    def layer(self, S=PREFILL_S):
        x = self._hidden(S)
        t0 = time.perf_counter()
        self.orc.layer(0, x, None, 0)
        return time.perf_counter() - t0

    def head(self, S=PREFILL_S):
        toks = self.si.tokens(1, S, 128256)
        x = self._hidden(S)
        t0 = time.perf_counter()
        self.orc.embed(toks)
        self.orc.logits(x[-1])
        return time.perf_counter() - t0

    def decode_layer(self, ctx=DECODE_CTX):
        si = self.si
        if self._cache is None:
            n = 8 * ctx * 128
            k = si.bf16_bits_to_f32(si.normal(3, si.STREAM_KV_BASE, n, 1.0, 'bf16')).reshape(8, ctx, 128)
            v = si.bf16_bits_to_f32(si.normal(3, si.STREAM_KV_BASE + 1, n, 1.0, 'bf16')).reshape(8, ctx, 128)
            self._cache = (k, v)
        c = self.SequenceCache(k=[self._cache[0]], v=[self._cache[1]])
        x = self._hidden(1)
        t0 = time.perf_counter()
        self.orc.layer(0, x, c, ctx)
        return time.perf_counter() - t0


def cpu_baseline(samples: OracleSample, layer_reps: int = 3) -> dict:
    """The oracle on the host cores (all BLAS threads, then one thread) for the
    prefill workload and for one decode step; about 20 s of CPU work."""
    from threadpoolctl import threadpool_limits
    cores = oracle_threads()
    t_layer = min(samples.layer() for _ in range(layer_reps))
    t_head = min(samples.head() for _ in range(2))
    t_dec = min(samples.decode_layer() for _ in range(5))
    t_dhead = min(samples.head(1) for _ in range(3))
    with threadpool_limits(limits=1, user_api='blas'):
        t1_layer = samples.layer(256)
        t1_head = samples.head(256)
    return {'value': PREFILL_S / (32 * t_layer + t_head), 'unit': 'tokens/s', 'cores': cores, 'kind': 'oracle',
            'sample': f'float32 numpy oracle, prefill B=1: one of the 32 layers at S={PREFILL_S} '
                      f'({t_layer:.3f} s, best of {layer_reps}) and the embedding + final norm + LM head of the '
                      f'last row ({t_head:.3f} s), each timed; value = {PREFILL_S} / (32 x layer + head)',
            'one_thread': {'value': 256 / (32 * t1_layer + t1_head), 'unit': 'tokens/s', 'cores': 1,
                           'sample': f'the same at S=256 with one BLAS thread (layer {t1_layer:.3f} s, '
                                     f'head {t1_head:.3f} s)'},
            'decode': {'value': 1.0 / (32 * t_dec + t_dhead), 'unit': 'tokens/s', 'cores': cores,
                       'sample': f'one decode step, B=1, context {DECODE_CTX} (N(0,1) cache): one layer '
                                 f'({t_dec * 1e3:.1f} ms, best of 5) x 32 plus the LM head of the row '
                                 f'({t_dhead * 1e3:.1f} ms)'}}


def workload_config(ws, args, NL=32):
    """The workload both arms report (the reference arm times a sample of it)."""
    return {'workload': 'llama3-8b-shape full-model prefill, B=1, S=2048 (32 layers + LM head '
                        '+ argmax); decode: B=32, context 4096, 128 greedy steps',
            'batch': PREFILL_B, 'seq_len': PREFILL_S, 'layers': NL,
            'l2': 'inputs larger than L2 (16 GB of weights streamed per step)',
            'parallelism': f'replicas x{ws}',
            'kv_cache': 'paged (128-position pages)' if args.paged else 'contiguous'}


def run_reference(args):
    """The oracle as the reference arm (the pages hold no implementation to
    install). Every step is one bounded sample: one of the 32 decoder layers
    of the 8B model over the B=1, S=2048 prompt; steps and ms_per_step describe
    exactly those timed samples. The line's value is the full-model prefill
    throughput derived from them and from the embedding + final norm + LM head
    of the last row, timed once in the same run."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    samples = OracleSample()
    for _ in range(args.warmup):
        samples.layer()
    times = [samples.layer() for _ in range(args.steps)]
    t_head = samples.head()
    dt = statistics.mean(times)
    cores = oracle_threads()
    value = PREFILL_S / (32 * dt + t_head)
    desc = (f'float32 numpy oracle; each step: one of the 32 layers of the 8B model at S={PREFILL_S} '
            f'(mean {dt:.3f} s); value = {PREFILL_S} / (32 x step + embedding/final-norm/LM-head time '
            f'{t_head:.3f} s)')
    line = {'impl': 'reference', 'metric': METRIC, 'value': value, 'unit': 'tokens/s', 'n_gpus': args.gpus,
            'steps': args.steps, 'warmup': args.warmup, 'ms_per_step': dt * 1e3, 'higher_is_better': True,
            'scaling': 'weak', 'vs_baseline': None, 'dtype': 'f32', 'data': 'synthetic (seeded)',
            'config': workload_config(ws, args),
            'cpu_baseline': {'value': value, 'unit': 'tokens/s', 'cores': cores, 'kind': 'oracle', 'sample': desc},
            'e2e': {'value': value, 'unit': 'tokens/s', 'h2d_bytes_per_step': 0, 'd2h_bytes_per_step': 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
D_, F_, H_, HK_, HD_, V_ = 4096, 14336, 32, 8, 128, 128256
# DRAM read + write bytes of one middle layer's chained launch (Wo, w1/w3,
# w2, next QKV) at B=1, S=2048, from an ncu capture of a 2-layer model of the
# 8B shapes. Other batches move other activation bytes: no figure for them.
PAIR_GEMM_TRAFFIC = 1096.8e6 + 163.6e6


def measure_prefill(L, m, st, toks, arg, args, ws, local, NL, tf_sust, peak_src, B=PREFILL_B):
    """Timed prefill steps of B sequences (no per-launch events), then the
    same steps with the library's per-launch events for the kernel breakdown
    and roofline."""
    import torch

    def prefill_step():
        L.llama_reset(m, st)
        L.llama_prefill(m, toks, B, PREFILL_S, st)
        L.llama_argmax(m, arg, st)

    for _ in range(args.warmup):
        prefill_step()
    torch.cuda.synchronize()
    assert L.llama_sync_status(m, st) == 0
    _barrier(ws)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = L.llama_kernel_launches()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        ev0.record(st)
        for _ in range(args.steps):
            prefill_step()
        ev1.record(st)
        torch.cuda.synchronize()
    launches = L.llama_kernel_launches() - n0
    _barrier(ws)
    ms = _max_over_ranks(ev0.elapsed_time(ev1) / args.steps, ws)
    L.llama_profile(m, 1)
    L.llama_profile_read(m)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(st)
    for _ in range(args.steps):
        prefill_step()
    p1.record(st)
    prof = L.llama_profile_read(m)
    L.llama_profile(m, 0)
    prof_ms = p0.elapsed_time(p1) / args.steps
    _barrier(ws)
    M = B * PREFILL_S
    flops_layer = 2.0 * M * D_ * ((H_ + 2 * HK_) * HD_ + H_ * HD_ + 2 * F_ + F_)
    gemm_kinds = ['gemm_qkv_rope', 'gemm_wo_residual', 'gemm_w13_swiglu', 'gemm_w2_residual', 'gemm_chain']
    gemm_ms = sum(prof[k][0] for k in gemm_kinds)
    gemm_launches = sum(prof[k][1] for k in gemm_kinds)
    achieved = flops_layer * NL * args.steps / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    total_prof = max(sum(x[0] for x in prof.values()), 1e-9)
    kernels = {k: {'ms_per_step': v[0] / args.steps, 'launches_per_step': v[1] / args.steps,
                   'share': v[0] / total_prof} for k, v in prof.items() if v[1]}
    attn_flops = 4.0 * B * H_ * HD_ * PREFILL_S * (PREFILL_S + 1) / 2 * NL
    attn = prof.get('attention_prefill', (0, 0))
    roofline = {'kernel': 'gemm_chain_kernel (tcgen05 cta_group::2; per layer one launch of Wo, w1/w3, w2 and the '
                          'next layer\'s QKV, plus layer 0\'s QKV)', 'bound': 'tensor',
                'achieved': achieved, 'peak': tf_sust, 'unit': 'TFLOP/s',
                'frac': achieved / tf_sust if achieved else None,
                'traffic': PAIR_GEMM_TRAFFIC if B == 1 else None,
                'traffic_note': ('DRAM read+write bytes of a middle layer\'s chained launch from one ncu capture '
                                 '(1.3x its operand bytes: w1/w3 weights stream twice by design, w2\'s weight is '
                                 'partly re-read per row block)') if B == 1 else
                                'not captured at this batch (the B=1 capture does not scale with the tokens)',
                'peak_kind': f'bf16 sustained ({peak_src}); fp16 has the same nominal tensor rate',
                'launches': gemm_launches // max(args.steps, 1),
                'attention_tflops': attn_flops * args.steps / (attn[0] / 1e3) / 1e12 if attn[0] else None,
                'measured': f'per-launch CUDA events on the launching stream over {args.steps} profiled steps '
                            f'({prof_ms:.2f} ms/step with events vs {ms:.2f} without)'}
    return ms, launches, clk.summary(), roofline, kernels


def measure_e2e(L, m, st, toks_h, args, ws):
    """The same prefill through llama_generate with pinned host buffers:
    host->device tokens, prefill, argmax, device->host next tokens, per step."""
    import torch
    host_toks = torch.from_numpy(toks_h.copy()).pin_memory()
    host_out = torch.empty(PREFILL_B, dtype=torch.int32).pin_memory()
    for _ in range(2):  # eager first call per shape, then the graph capture
        L.llama_reset(m, st)
        L.llama_generate(m, host_toks, PREFILL_B, PREFILL_S, 0, host_out, st)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    e0.record(st)
    for _ in range(args.steps):
        L.llama_reset(m, st)
        L.llama_generate(m, host_toks, PREFILL_B, PREFILL_S, 0, host_out, st)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_value, _ = replica_throughput(PREFILL_B * PREFILL_S, e0.elapsed_time(e1) / args.steps, ws)
    return {'value': e2e_value, 'unit': 'tokens/s',
            'h2d_bytes_per_step': PREFILL_B * PREFILL_S * 4, 'd2h_bytes_per_step': PREFILL_B * 4,
            'api': 'llama_generate(host tokens, n_new=0)'}


def measure_decode(L, m, st, arg, args, ws, local, NL, hbm_peak, peak_src):
    """Batch-32 greedy decode over a 4096-token cache: 128 graph-replayed steps,
    then 8 eager steps with per-launch events for the breakdown."""
    import numpy as np
    import torch
    import seeded_inputs as si
    L.llama_fill_kv_random(m, 3, DECODE_CTX, st)
    first = torch.from_numpy(si.tokens(1, DECODE_B, V_, start=PREFILL_B * PREFILL_S)).cuda()
    lens = np.full(DECODE_B, DECODE_CTX, np.int32)

    def decode_run(n):
        L.llama_set_lengths(m, lens, DECODE_B, st)
        cur = first
        for _ in range(n):
            L.llama_decode_step(m, cur, DECODE_B, st)
            L.llama_argmax(m, arg, st)
            cur = arg

    decode_run(max(args.warmup, 2))  # eager first call, then graph capture
    torch.cuda.synchronize()
    _barrier(ws)
    L.llama_set_lengths(m, lens, DECODE_B, st)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = first
    n0 = L.llama_kernel_launches()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        d0.record(st)
        for _ in range(DECODE_STEPS):
            L.llama_decode_step(m, cur, DECODE_B, st)
            L.llama_argmax(m, arg, st)
            cur = arg
        d1.record(st)
        torch.cuda.synchronize()
    launches = L.llama_kernel_launches() - n0
    dvalue, dms = replica_throughput(DECODE_B, d0.elapsed_time(d1) / DECODE_STEPS, ws)
    assert L.llama_sync_status(m, st) == 0
    L.llama_profile(m, 1)
    L.llama_profile_read(m)
    decode_run(8)
    dprof = L.llama_profile_read(m)
    L.llama_profile(m, 0)
    avg_ctx = DECODE_CTX + (DECODE_STEPS + 1) / 2.0
    w_bytes = NL * 2.0 * (D_ * (H_ + 2 * HK_) * HD_ + D_ * H_ * HD_ + 2 * D_ * F_ + D_ * F_) + 2.0 * V_ * D_
    kv_bytes = NL * 2.0 * DECODE_B * avg_ctx * HK_ * HD_ * 2
    step_bytes = w_bytes + kv_bytes
    achieved = step_bytes / (dms / 1e3) / 1e9
    return {'value': dvalue, 'unit': 'tokens/s', 'ms_per_step': dms,
            'steps': DECODE_STEPS, 'batch': DECODE_B, 'context': DECODE_CTX, 'graph_replay': True,
            'gpu_launches': launches,
            'roofline': {'bound': 'hbm', 'achieved': achieved, 'peak': hbm_peak, 'unit': 'GB/s',
                         'frac': achieved / hbm_peak, 'traffic': None, 'algorithmic_bytes_per_step': step_bytes,
                         'peak_kind': f'hbm copy ({peak_src})'},
            'kernels_eager_profile': {k: {'ms_per_step': v[0] / 8, 'launches_per_step': v[1] / 8}
                                      for k, v in dprof.items() if v[1]},
            'clocks': clk.summary()}


def measure_block(L, m, st, S, args, hbm_peak, tf_burst, tf_sust, peak_src):
    """One 8B-shaped decoder block (layer 0 of the model) on N(0,1) hidden
    states of one sequence of S tokens at positions 0..S-1: S = 17 is bound by
    streaming the block's 436 MB of weights, S = 2048 by the tensor cores.
    Weights (436 MB) exceed L2, so every call streams them from HBM."""
    import torch
    x = torch.empty((1, S, D_), dtype=torch.float32, device='cuda')
    L.llama_fill_normal(x, x.numel(), 2, (1 << 20) + 1, 1.0, L.LLAMA_F32, st)
    y = torch.empty_like(x)
    lens = __import__('numpy').zeros(DECODE_B, __import__('numpy').int32)
    L.llama_set_lengths(m, lens, DECODE_B, st)
    for _ in range(max(args.warmup, 3)):
        L.llama_block_forward(m, 0, x, y, 1, S, st)
    torch.cuda.synchronize()
    reps = max(args.steps, 10)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(reps):
        L.llama_block_forward(m, 0, x, y, 1, S, st)
    e1.record(st)
    torch.cuda.synchronize()
    assert L.llama_sync_status(m, st) == 0
    ms = e0.elapsed_time(e1) / reps
    w_bytes = 2.0 * (D_ * (H_ + 2 * HK_) * HD_ + D_ * H_ * HD_ + 3 * D_ * F_)
    flops = 2.0 * S * w_bytes / 2 + 4.0 * H_ * HD_ * S * (S + 1) / 2
    out = {'value': S / (ms / 1e3), 'unit': 'tokens/s', 'ms_per_call': ms, 'calls': reps,
           'workload': f'one 8B-shaped decoder block, B=1, S={S}, positions 0..{S - 1}, N(0,1) hidden states'}
    if S <= 128:
        gbs = w_bytes / (ms / 1e3) / 1e9
        out['roofline'] = {'bound': 'hbm', 'achieved': gbs, 'peak': hbm_peak, 'unit': 'GB/s',
                           'frac': gbs / hbm_peak, 'work': 'weight bytes per call (activations negligible)',
                           'peak_kind': f'hbm copy ({peak_src})'}
    else:
        tf = flops / (ms / 1e3) / 1e12
        out['roofline'] = {'bound': 'tensor', 'achieved': tf, 'peak': tf_burst, 'unit': 'TFLOP/s',
                           'frac': tf / tf_burst, 'work': 'linear + causal attention flops per call',
                           'peak_kind': f'bf16 burst ({peak_src}): the block is timed alone'}
    return out


def measure_long(L, st, args, tf_burst, peak_src):
    """Long-context prefill through one 8B-shaped decoder layer: 32768
    positions of one sequence fed through llama_block_forward in 4096-token
    chunks, each chunk's queries attending to every earlier chunk's keys in
    the cache (N(0,1) hidden states; a separate one-layer model with a
    32768-position cache). Causal attention is ~38% of the flops here against
    ~4% at 2048 tokens."""
    import numpy as np
    import torch
    from llama_transformer_decoder_b200.configs import LLAMA3_8B, make_config
    cfg = make_config(LLAMA3_8B, dtype=L.LLAMA_BF16, max_batch=1, max_seq=LONG_S, max_tokens=LONG_CHUNK, n_layers=1)
    m2 = L.llama_create(cfg)
    try:
        L.llama_init_weights(m2, 0, 0.02, st)
        x = torch.empty((1, LONG_CHUNK, D_), dtype=torch.float32, device='cuda')
        L.llama_fill_normal(x, x.numel(), 2, (1 << 20) + 2, 1.0, L.LLAMA_F32, st)
        y = torch.empty_like(x)

        def one_pass():
            for a in range(0, LONG_S, LONG_CHUNK):
                L.llama_set_lengths(m2, np.array([a], np.int32), 1, st)
                L.llama_block_forward(m2, 0, x, y, 1, LONG_CHUNK, st)

        one_pass()
        torch.cuda.synchronize()
        reps = max(2, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(reps):
            one_pass()
        e1.record(st)
        torch.cuda.synchronize()
        assert L.llama_sync_status(m2, st) == 0
        ms = e0.elapsed_time(e1) / reps
    finally:
        L.llama_destroy(m2)
    w_elems = D_ * (H_ + 2 * HK_) * HD_ + D_ * H_ * HD_ + 3 * D_ * F_
    lin = 2.0 * LONG_S * w_elems
    attn = 4.0 * H_ * HD_ * LONG_S * (LONG_S + 1) / 2
    tf = (lin + attn) / (ms / 1e3) / 1e12
    return {'value': LONG_S / (ms / 1e3), 'unit': 'tokens/s', 'ms_per_pass': ms, 'passes': reps,
            'workload': f'one 8B-shaped decoder layer, B=1, {LONG_S} positions in {LONG_CHUNK}-token chunks '
                        '(chunked prefill over the cache), N(0,1) hidden states',
            'attention_share_of_flops': attn / (lin + attn),
            'roofline': {'bound': 'tensor', 'achieved': tf, 'peak': tf_burst, 'unit': 'TFLOP/s', 'frac': tf / tf_burst,
                         'work': 'linear + causal attention flops per pass',
                         'peak_kind': f'bf16 burst ({peak_src}): one layer timed alone'}}


def run_ours(args):
    import torch
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        import torch.distributed as dist
        dist.init_process_group('nccl', timeout=datetime.timedelta(seconds=600), device_id=torch.device('cuda', local))
    from llama_transformer_decoder_b200 import binding as L
    from llama_transformer_decoder_b200.configs import LLAMA3_8B, make_config
    import seeded_inputs as si
    hbm_peak, tf_burst, tf_sust, peak_src = _peaks()

    NL = args.layers
    max_seq = DECODE_CTX + DECODE_STEPS + max(args.warmup, 2) + 8
    cfg = make_config(LLAMA3_8B, dtype=L.LLAMA_BF16, max_batch=DECODE_B, max_seq=max_seq,
                      max_tokens=PREFILL_B8 * PREFILL_S, n_layers=NL, kv_page_size=128 if args.paged else 0)
    st = torch.cuda.Stream()
    m = L.llama_create(cfg)
    L.llama_init_weights(m, 0, 0.02, st)
    toks_h = si.tokens(1, PREFILL_B * PREFILL_S, V_).reshape(PREFILL_B, PREFILL_S)
    toks = torch.from_numpy(toks_h).cuda()
    arg = torch.empty(DECODE_B, dtype=torch.int32, device='cuda')
    torch.cuda.synchronize()

    ms = launches = clk = roofline = kernels = e2e = None
    prefill_b8 = blocks = long_prefill = None
    if not args.decode_only:
        ms, launches, clk, roofline, kernels = measure_prefill(L, m, st, toks, arg, args, ws, local, NL, tf_sust,
                                                               peak_src)
        e2e = measure_e2e(L, m, st, toks_h, args, ws)
        if not args.no_extra:
            toks8 = torch.from_numpy(si.tokens(1, PREFILL_B8 * PREFILL_S, V_).reshape(PREFILL_B8, PREFILL_S)).cuda()
            ms8, _, clk8, roof8, _ = measure_prefill(L, m, st, toks8, arg, args, ws, local, NL, tf_sust, peak_src,
                                                     B=PREFILL_B8)
            v8, _ = replica_throughput(PREFILL_B8 * PREFILL_S, ms8, ws)
            prefill_b8 = {'value': v8, 'unit': 'tokens/s', 'ms_per_step': ms8, 'batch': PREFILL_B8,
                          'seq_len': PREFILL_S, 'roofline': roof8, 'clocks': clk8}
            blocks = {f's{S}': measure_block(L, m, st, S, args, hbm_peak, tf_burst, tf_sust, peak_src)
                      for S in (17, 2048)}
            long_prefill = measure_long(L, st, args, tf_burst, peak_src)
    decode = None if args.no_decode else measure_decode(L, m, st, arg, args, ws, local, NL, hbm_peak, peak_src)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and NL == 32 and not args.decode_only:
        cpu = cpu_baseline(OracleSample())
    L.llama_destroy(m)
    if rank == 0:
        value = ws * PREFILL_B * PREFILL_S / (ms / 1e3) if ms else None
        line = {'metric': METRIC, 'value': value, 'unit': 'tokens/s', 'n_gpus': ws, 'steps': args.steps,
                'warmup': args.warmup, 'ms_per_step': ms, 'higher_is_better': True, 'scaling': 'weak',
                'vs_baseline': None, 'dtype': 'f16',
                'data': 'synthetic: seeded N(0,0.02) weights of the 8B shapes rounded to bf16 (held as fp16), '
                        'uniform token ids',
                'config': workload_config(ws, args, NL),
                'roofline': roofline, 'cpu_baseline': cpu, 'e2e': e2e, 'gpu_launches': launches,
                'clocks': clk, 'kernels': kernels, 'decode': decode, 'prefill_b8': prefill_b8,
                'block_8b': blocks, 'long_prefill': long_prefill}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------ one kernel
def run_kernel(args):
    """One kernel alone on seeded fp16 inputs from the library's device
    generator (for ncu captures and shape sweeps): prints one JSON line per
    shape with its CUDA-event time per call (median over --steps calls, L2
    flushed by a 256 MB write enqueued before each) and its rate against the
    burst peaks (it runs alone). --batch, --seq and --ctx take comma-separated
    lists."""
    import torch
    from llama_transformer_decoder_b200 import binding as L
    torch.cuda.set_device(0)
    hbm, tf_burst, _, src = _peaks()
    F16 = L.LLAMA_F16
    dev = 'cuda'

    def filled(shape, stream_id, std=1.0):
        t = torch.empty(shape, dtype=torch.float16, device=dev)
        L.llama_fill_normal(t, t.numel(), 9, stream_id, std, F16)
        return t

    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MB > L2
    H, Hk, d = 32, 8, 128
    ints = lambda v: [int(x) for x in str(v).split(',')]
    cases = []
    if args.kernel == 'attention_prefill':
        cases = [(B, S) for B in ints(args.batch) for S in ints(args.seq)]
    elif args.kernel == 'attention_decode':
        cases = [(B, C) for B in ints(args.batch) for C in ints(args.ctx)]
    else:
        cases = [tuple(int(x) for x in args.mnk.split(','))]
    for case in cases:
        if args.kernel == 'attention_prefill':
            B, S = case
            q, k, v = filled((B, H, S, d), 1), filled((B, Hk, S, d), 2), filled((B, Hk, S, d), 3)
            o = torch.empty((B, S, H * d), dtype=torch.float16, device=dev)
            call = lambda: L.llama_attention_prefill(q, k, v, o, B, S, H, Hk, d, F16)
            work, unit, peak = 4.0 * B * H * d * S * (S + 1) / 2, 'TFLOP/s', tf_burst
            cfg = {'workload': f'causal GQA prefill attention B={B} S={S} H=32 Hk=8 d=128'}
        elif args.kernel == 'attention_decode':
            B, C = case
            q, kc, vc = filled((B, H, d), 1), filled((B, Hk, C, d), 2), filled((B, Hk, C, d), 3)
            ln = torch.full((B,), C, dtype=torch.int32, device=dev)
            o = torch.empty((B, H * d), dtype=torch.float16, device=dev)
            call = lambda: L.llama_attention_decode(q, kc, vc, ln, o, B, C, H, Hk, d, F16)
            work, unit, peak = float(B * Hk * C * d * 2 * 2), 'GB/s', hbm
            cfg = {'workload': f'decode attention B={B} context={C} H=32 Hk=8 d=128'}
        else:
            M, N, K = case
            x, w = filled((M, K), 1), filled((N, K), 2, 0.02)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            call = lambda: L.llama_linear(x, w, y, M, N, K, F16, 0)
            if M <= 128:
                work, unit, peak = float(N * K * 2), 'GB/s', hbm
            else:
                work, unit, peak = 2.0 * M * N * K, 'TFLOP/s', tf_burst
            cfg = {'workload': f'linear y = x W^T, M={M} N={N} K={K}'}
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        times = []
        for _ in range(args.steps):
            # The flush is enqueued, not waited for: the call is launched while
            # the GPU still writes the flush buffer, so the host's launch work
            # never shows as device idle time between the two events.
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.add_(1.0)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        assert L.llama_status(None) == 0
        ms = statistics.median(times)
        rate = work / (ms / 1e3) / (1e12 if unit == 'TFLOP/s' else 1e9)
        print(json.dumps({'kernel': args.kernel, 'ms': ms, 'rate': rate, 'unit': unit, 'peak': peak,
                          'frac': rate / peak, 'peak_kind': f'burst ({src})', 'steps': args.steps,
                          'warmup': args.warmup, 'config': cfg}), flush=True)
        del call
        torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument('--gpus', type=int, default=1)
    ap.add_argument('--steps', type=int, default=5)
    ap.add_argument('--warmup', type=int, default=3)
    ap.add_argument('--impl', choices=['ours', 'reference'], default='ours')
    ap.add_argument('--no-decode', action='store_true')
    ap.add_argument('--decode-only', action='store_true', help='skip the prefill and end-to-end legs (profiling)')
    ap.add_argument('--layers', type=int, default=32, help='decoder layers (32 = the 8B model)')
    ap.add_argument('--no-cpu-baseline', action='store_true')
    ap.add_argument('--no-extra', action='store_true', help='skip the B=8 prefill and single-block legs')
    ap.add_argument('--paged', action='store_true', help='run the model with the paged KV cache')
    ap.add_argument('--kernel', choices=['attention_prefill', 'attention_decode', 'linear'],
                    help='time one kernel alone on seeded inputs (profiling and sweeps)')
    ap.add_argument('--batch', default='1', help='--kernel attention_*: sequences (comma list)')
    ap.add_argument('--seq', default='2048', help='--kernel attention_prefill: tokens per sequence (comma list)')
    ap.add_argument('--ctx', default='4096', help='--kernel attention_decode: cached keys (comma list)')
    ap.add_argument('--mnk', default='2048,28672,4096', help='--kernel linear: M,N,K')
    args = ap.parse_args()
    if args.kernel:
        return run_kernel(args)
    if args.impl == 'reference':
        return run_reference(args)
    return run_ours(args)


if __name__ == '__main__':
    sys.exit(main())
