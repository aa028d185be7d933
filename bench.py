#!/usr/bin/env python
"""Benchmark of the TurboQuant codec on B200.

Step (timed unit): encode then decode the K and V tensors of one Llama-style
KV-cache layer [8, 8192, 8, 128] fp16 at 2, 3 and 4 bits. K and V are stored
together in one [2, 524288, 128] buffer, as a serving engine's KV cache is,
so each width is one tq_encode and one tq_decode call over both tensors: 6
kernel launches, each on buffers not touched by the previous launch (256 MiB
of fp16 per launch, larger than L2).

value = fp16-equivalent bytes of the step (2 * d bytes per vector per encode
or decode) / device time of the step, aggregated over ranks (weak scaling:
each rank codes its own layer). The same JSON line carries the fused
decode-step attention ("attn": 16 query tokens over 32768-position packed
caches, K 4 bits / V 2 bits) and the streaming append ("append": 256
sequences x 8 heads per step), each timed in its own loop, the roofline of
the dominant kernel, the oracle CPU baseline, clocks and an end-to-end figure
through the public API with host buffers.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

D = 128
LAYER = (8, 8192, 8, 128)
BITS = (2, 3, 4)
ATTN = dict(B=16, Hq=32, Hkv=8, S=32768, d=128, kb=4, vb=2)
APPEND = dict(n_seq=256, H=8, d=128, bits=4, s_max=1024)
L2_BYTES = 126 * 1024 * 1024


HBM_NOMINAL_GBS = 8000.0  # B200 nominal HBM3e bandwidth, printed beside the measured copy peak
FP32_LANES_PER_SM = 128   # FP32 FMA lanes per SM (4 sub-partitions x 32)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, with_power: bool = False):
        self.idx = gpu_index
        self.with_power = with_power
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"tq_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for ln in open(self.path):
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                try:
                    pw.append(float(parts[3]))
                except ValueError:
                    pass
                for name, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(name)
            os.remove(self.path)
        except Exception:
            pass
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
               "samples": len(sm), "reasons": sorted(reasons)}
        if self.with_power:
            out["power_w"] = statistics.median(pw) if pw else None
        return out


def _source_hash(name: str) -> str:
    with open(os.path.join(ROOT, "kv_cache_vector_turboquant_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def _profile_traffic(kernel_file: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    has not changed since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    vals = {}
    for ln in open(path):
        if ":" in ln:
            k, v = ln.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != _source_hash(kernel_file):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def _ev(torch):
    return torch.cuda.Event(enable_timing=True)


def _bracketed_ms(torch, call, steps):
    """Mean ms per call over `steps` back-to-back calls between two events
    (no event between the calls, which would serialise them)."""
    t0, t1 = _ev(torch), _ev(torch)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(steps):
        call()
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def reduce_max_ms(ms: float, world: int, dist=None, device=None) -> float:
    """Max over ranks of a per-rank time (the slowest rank sets the job time)."""
    if world <= 1:
        return ms
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step_per_rank: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job GB/s: the bytes all ranks processed / the max-over-ranks time."""
    return bytes_per_step_per_rank * steps * world / (ms_max / 1e3) / 1e9


def _codec_step_setup(K, W, torch, rank):
    """Buffers and the 6 launches of one step (closures on the current stream).

    The layer's K and V live in one [2, n, d] buffer (the layout of a serving
    engine's KV cache, [2, ...]), so each width takes one tq_encode and one
    tq_decode call over both tensors (2n rows); `xs`, `packed` and `norms`
    also give per-tensor views."""
    k, v = W.llama_layer(device="cuda", k_seed=1 + 100 * rank, v_seed=2 + 100 * rank)
    n = k.numel() // D
    kv = torch.stack([k.reshape(n, D), v.reshape(n, D)])  # [2, n, d]
    del k, v
    xs = {"K": kv[0], "V": kv[1]}
    codecs = {b: K.TurboQuant(D, b) for b in BITS}
    packed_kv = {b: torch.empty(2, n, codecs[b].packed_bytes, dtype=torch.uint8, device="cuda") for b in BITS}
    norms_kv = {b: torch.empty(2, n, dtype=torch.float32, device="cuda") for b in BITS}
    packed = {(b, t): packed_kv[b][i] for b in BITS for i, t in enumerate("KV")}
    norms = {(b, t): norms_kv[b][i] for b in BITS for i, t in enumerate("KV")}
    out_kv = torch.empty(2, n, D, dtype=torch.float16, device="cuda")
    launches = []  # (kind, bits, fn, algorithmic bytes, fp16-equivalent bytes)
    for b in BITS:
        alg = 2 * n * (2 * D + codecs[b].packed_bytes + 4)
        launches.append(("encode", b, (lambda b=b: K.tq_encode(codecs[b].ctx, kv, 2 * n, packed_kv[b], norms_kv[b])),
                         alg, 2 * 2 * D * n))
    for b in BITS:
        alg = 2 * n * (2 * D + codecs[b].packed_bytes + 4)
        launches.append(("decode", b, (lambda b=b: K.tq_decode(codecs[b].ctx, packed_kv[b], norms_kv[b], 2 * n,
                                                               out_kv)), alg, 2 * 2 * D * n))
    return dict(n=n, xs=xs, codecs=codecs, packed=packed, norms=norms, out=out_kv[0], launches=launches)


def _bench_attention(K, W, torch, steps, warmup, sm_mhz=1965.0):
    a = ATTN
    q, k, v = W.decode_step(a["B"], a["Hq"], a["Hkv"], a["S"], a["d"])
    kc, vc = K.TurboQuant(a["d"], a["kb"]), K.TurboQuant(a["d"], a["vb"])
    kp, kn = kc.encode(k)
    vp, vn = vc.encode(v)
    del k, v
    pos = torch.full((a["B"],), a["S"], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    wsb = K.tq_attend_workspace_bytes(a["B"], a["Hq"], a["d"], a["S"])
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")

    def call():
        K.tq_attend_decode(kc.ctx, vc.ctx, q, a["B"], a["Hq"], a["Hkv"], kp, kn, vp, vn, a["S"], pos, out, ws, wsb)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    evs = [(_ev(torch), _ev(torch)) for _ in range(steps)]
    for e0, e1 in evs:
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]  # per step, with events around each
    t = _bracketed_ms(torch, call, steps) / 1e3    # back-to-back steps
    pk, pv = a["d"] * a["kb"] // 8, a["d"] * a["vb"] // 8
    alg = a["B"] * a["S"] * a["Hkv"] * (pk + pv + 8) + 2 * 2 * a["B"] * a["Hq"] * a["d"]
    peak, kind = _peaks()
    ach = alg / t / 1e9
    g = a["Hq"] // a["Hkv"]
    flops = 4 * g * a["d"] * a["B"] * a["S"] * a["Hkv"]
    fp32_peak = torch.cuda.get_device_properties(0).multi_processor_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6
    st = K.tq_device_error()
    paged = _bench_attention_paged(K, torch, a, q, kc, vc, kp, kn, vp, vn, pos, steps, warmup, alg)
    return {"workload": "decode_step: q [16,32,128] fp16, K 4-bit / V 2-bit packed caches [16,32768,8,*]",
            "tokens_per_s": a["B"] / t, "ms_per_step": t * 1e3, "ms_median": statistics.median(ms),
            "cache_positions_heads_per_s": a["B"] * a["S"] * a["Hkv"] / t,
            "launches_per_step": 2,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                         "frac_of_nominal": ach / HBM_NOMINAL_GBS,
                         "traffic": _profile_traffic("tq_attend_fast.cu", "attend_fast_decode_step.txt"),
                         "peak_kind": kind, "algorithmic_bytes": alg},
            # 2 g d multiply-adds per (position, kv head), g = Hq / Hkv: on the
            # FP32 pipes (SMs x 128 lanes x 2 flop per cycle) this step could
            # not beat `fp32_bound_us`; the kernel runs both contractions on
            # the tensor cores instead
            "flops": flops, "fp32_bound_us": flops / fp32_peak * 1e6, "fp32_peak_tflops": fp32_peak / 1e12,
            "device_error": list(st), "paged": paged}


def _bench_attention_paged(K, torch, a, q, kc, vc, kp, kn, vp, vn, pos, steps, warmup, alg):
    """The same decode step over a paged cache: the 16-position blocks of all
    sequences scattered over the pool by a random permutation, read through
    block tables [16, 2048]."""
    B, S = a["B"], a["S"]
    nb = S // 16
    perm = torch.randperm(B * nb, generator=torch.Generator().manual_seed(3)).cuda()

    def pages(t):
        blocks = t.reshape(B * nb, 16, *t.shape[2:])
        pool = torch.empty_like(blocks)
        pool[perm] = blocks
        return pool

    kpool, knpool, vpool, vnpool = pages(kp), pages(kn), pages(vp), pages(vn)
    bt = perm.reshape(B, nb).to(torch.int32)
    out = torch.empty_like(q)
    wsb = K.tq_attend_workspace_bytes(B, a["Hq"], a["d"], S)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")

    def call():
        K.tq_attend_decode_paged(kc.ctx, vc.ctx, q, B, a["Hq"], a["Hkv"], kpool, knpool, vpool, vnpool, B * nb, bt,
                                 nb, pos, out, ws, wsb)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    evs = [(_ev(torch), _ev(torch)) for _ in range(steps)]
    for e0, e1 in evs:
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    t = _bracketed_ms(torch, call, steps) / 1e3
    peak, kind = _peaks()
    st = K.tq_device_error()
    del kpool, knpool, vpool, vnpool
    return {"workload": "decode_step over a paged cache: 16-position blocks scattered by a random permutation, "
                        "block tables [16, 2048]",
            "tokens_per_s": B / t, "ms_per_step": t * 1e3, "GBps": alg / t / 1e9, "frac": alg / t / 1e9 / peak,
            "device_error": list(st)}


def _bench_append(K, W, torch, steps_per_run=1024):
    """Streaming append: K and V of 256 sequences x 8 heads, one token per
    step for 1024 steps into a preallocated [256, 1024, 8, P] cache, at every
    head_dim x width, written by two tq_encode_append calls per step and by
    one tq_encode_append_kv call (`fused_` keys). Per-step latency from
    events around each eager step; the same 1024 steps are then captured once
    in a CUDA graph and replayed, which removes the host launch cost."""
    res = {}
    for d in (64, 128, 256):
        for b in BITS:
            c = K.TurboQuant(d, b)
            P = c.packed_bytes
            n_seq, H, s_max = APPEND["n_seq"], APPEND["H"], steps_per_run
            toks = W.append_stream(run=d * 10 + b, steps=steps_per_run, n_seq=n_seq, H=H, d=d)
            cache = {t: torch.empty(n_seq, s_max, H, P, dtype=torch.uint8, device="cuda") for t in "KV"}
            cn = {t: torch.empty(n_seq, s_max, H, dtype=torch.float32, device="cuda") for t in "KV"}
            slots = torch.arange(s_max, dtype=torch.int32, device="cuda")[:, None].expand(s_max, n_seq).contiguous()

            def two(s):  # K and V with one tq_encode_append each
                for t in "KV":
                    K.tq_encode_append(c.ctx, toks[s], n_seq, H, cache[t], cn[t], s_max, slots[s])

            def fused(s):  # K and V in one tq_encode_append_kv launch
                K.tq_encode_append_kv(c.ctx, toks[s], toks[s], n_seq, H, cache["K"], cn["K"], cache["V"], cn["V"],
                                      s_max, slots[s])

            byts = steps_per_run * 2 * n_seq * H * (2 * d + P + 4)
            row = {}
            for name, one in (("", two), ("fused_", fused)):
                for s in range(8):
                    one(s)
                torch.cuda.synchronize()
                evs = [(_ev(torch), _ev(torch)) for _ in range(steps_per_run)]
                for s, (e0, e1) in enumerate(evs):
                    e0.record()
                    one(s)
                    e1.record()
                torch.cuda.synchronize()
                ms = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
                total = sum(ms) / 1e3
                # the whole stream of steps as one CUDA graph (every launch
                # was made once above, so its one-time set-up is done)
                g_stream = torch.cuda.Stream()
                g_stream.wait_stream(torch.cuda.current_stream())
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.stream(g_stream):
                    with torch.cuda.graph(graph, stream=g_stream):
                        for s in range(steps_per_run):
                            one(s)
                torch.cuda.current_stream().wait_stream(g_stream)
                graph.replay()
                torch.cuda.synchronize()
                g0, g1 = _ev(torch), _ev(torch)
                g0.record()
                graph.replay()
                g1.record()
                torch.cuda.synchronize()
                g_total = g0.elapsed_time(g1) / 1e3
                row.update({f"{name}p50_us": ms[len(ms) // 2] * 1e3, f"{name}p99_us": ms[int(len(ms) * 0.99) - 1] * 1e3,
                            f"{name}GBps": byts / total / 1e9,
                            f"{name}graph_us_per_step": g_total / steps_per_run * 1e6,
                            f"{name}graph_GBps": byts / g_total / 1e9})
                del graph
            res[f"d{d}_b{b}"] = row
            del cache, cn, toks
    res["launches_per_step"] = {"two_calls": 2, "fused": 1}
    res["steps"] = steps_per_run
    return res


def _bench_offset_variant(K, W, torch, reps=10):
    """The offset + fp16-scale variant (4 bits) on the llama layer's K and V
    tensors, alternating, one launch per tensor: encode, then decode."""
    k, v = W.llama_layer(device="cuda")
    xs = [k.reshape(-1, D), v.reshape(-1, D)]
    n = xs[0].shape[0]
    c = K.TurboQuant(D, 4)
    P = c.packed_bytes
    pk = [torch.empty(n, P, dtype=torch.uint8, device="cuda") for _ in xs]
    sd = [torch.empty(n, dtype=torch.int32, device="cuda") for _ in xs]
    out = [torch.empty(n, D, dtype=torch.float16, device="cuda") for _ in xs]
    for i in range(4):
        K.tq_encode_os(c.ctx, xs[i % 2], n, pk[i % 2], sd[i % 2])
        K.tq_decode_os(c.ctx, pk[i % 2], sd[i % 2], n, out[i % 2])
    torch.cuda.synchronize()
    res = {}
    peak, kind = _peaks()
    alg = n * (2 * D + P + 4)
    for name, fn in (("encode", lambda i: K.tq_encode_os(c.ctx, xs[i % 2], n, pk[i % 2], sd[i % 2])),
                     ("decode", lambda i: K.tq_decode_os(c.ctx, pk[i % 2], sd[i % 2], n, out[i % 2]))):
        e0, e1 = _ev(torch), _ev(torch)
        e0.record()
        for i in range(reps):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / reps / 1e3
        res[name] = {"us": t * 1e6, "GBps": alg / t / 1e9, "frac": alg / t / 1e9 / peak}
    res["workload"] = "offset + fp16-scale variant, 4 bits, llama layer K/V [8,8192,8,128] (one tensor per launch)"
    res["device_error"] = list(K.tq_device_error())
    del k, v, xs, pk, sd, out
    return res


def _bench_long_context(K, W, torch, reps=2):
    """The 80-layer long-context cache at 3 bits: K and V [1, 131072, 8, 128]
    of every layer, all resident in HBM (each layer's K and V in one buffer),
    encoded layer by layer on one stream: 80 launches of 2,097,152 vectors,
    42.9 GB of fp16 input. Data generation is not timed."""
    n_layers, S, H, d, bits = 80, 131072, 8, 128, 3
    c = K.TurboQuant(d, bits)
    P = c.packed_bytes
    scales = W.long_context_scales(n_layers, H, d)
    xs = []  # per layer, K and V in one [2 S H, d] buffer (one call per layer)
    for layer in range(n_layers):
        kx, vx = W.long_context_layer(layer, S, H, d, scales=scales)
        xs.append(torch.cat([kx.reshape(-1, d), vx.reshape(-1, d)]))
        del kx, vx
    n = 2 * S * H
    packed = [torch.empty(n, P, dtype=torch.uint8, device="cuda") for _ in xs]
    norms = [torch.empty(n, dtype=torch.float32, device="cuda") for _ in xs]

    def run():
        for x, p, nr in zip(xs, packed, norms):
            K.tq_encode(c.ctx, x, n, p, nr)

    run()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = _ev(torch), _ev(torch)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    t = min(times)
    alg = len(xs) * n * (2 * d + P + 4)
    peak, kind = _peaks()
    st = K.tq_device_error()
    out = {"workload": "long_context: 80 layers x K,V [1,131072,8,128] fp16, encode at 3 bits, layer by layer "
                       "(K and V of a layer in one call)",
           "ms": t * 1e3, "input_GB": len(xs) * n * 2 * d / 1e9, "launches": len(xs),
           "fp16_equiv_GBps": len(xs) * n * 2 * d / t / 1e9, "GBps": alg / t / 1e9, "frac": alg / t / 1e9 / peak,
           "vectors_per_s": len(xs) * n / t, "reps": reps, "device_error": list(st)}
    del xs, packed, norms
    torch.cuda.empty_cache()
    return out


LLAMA_WORKLOAD = ("llama_layer: K and V fp16 [8,8192,8,128] (K with 4 x10 channels per head) in one [2,...] "
                  "buffer, encode+decode at bits 2,3,4")


def _oracle_cores() -> int:
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def _loaded_native_libs() -> list:
    """Shared libraries of this repository mapped into this process."""
    out = set()
    try:
        with open("/proc/self/maps") as f:
            for ln in f:
                path = ln.split()[-1] if ln.strip() else ""
                if path.startswith(ROOT) and ".so" in os.path.basename(path):
                    out.add(os.path.relpath(path, ROOT))
    except OSError:
        pass
    return sorted(out)


def _oracle_sample(rows: int, seed: int):
    """`rows` random rows of each of the layer's K and V tensors (same rows),
    generated on the host (the oracle arm touches no GPU)."""
    import torch

    import tq_workloads as W

    k, v = W.llama_layer(device="cpu")
    fk, fv = k.reshape(-1, D), v.reshape(-1, D)
    idx = torch.randperm(fk.shape[0], generator=torch.Generator().manual_seed(seed))[:rows]
    return fk[idx].numpy(), fv[idx].numpy()


def _oracle_step(xk, xv) -> int:
    """One pass of the benchmarked step on a sample: encode and decode of the
    K and V rows at 2, 3 and 4 bits. Returns its fp16-equivalent bytes."""
    import oracle as O

    for bits in BITS:
        for xs in (xk, xv):
            p, nrm = O.encode(xs, bits, 42)
            O.decode(p, nrm, bits, 42, D)
    return len(BITS) * 2 * 2 * (2 * D) * (len(xk))


def _ordered_f16(h):
    """fp16 bit patterns -> integers ordered like the values (+0 == -0)."""
    import numpy as np

    u = np.asarray(h, dtype=np.float16).view(np.uint16).astype(np.int32)
    return np.where(u & 0x8000, -(u & 0x7FFF), u)


class _ParityTally:
    """The GPU's outputs for sampled rows of the benchmarked tensors against
    the oracle's: code mismatches (and how many of them lie outside the 1e-5
    boundary band), the largest relative norm error and the largest fp16 ulp
    distance between the GPU decode of the GPU's bytes and the oracle decode
    of the same bytes, per width and tensor."""

    def __init__(self):
        self.t = {}

    def add(self, bits, name, det, gp, gn, gx):
        import numpy as np

        import oracle as O

        r = self.t.setdefault(f"{name}_b{bits}", {"coords_checked": 0, "boundary_mismatches": 0,
                                                  "mismatches_outside_band": 0, "max_norm_rel_err": 0.0,
                                                  "max_decode_ulp": 0})
        gi = O.unpack_codes(gp, bits, D)
        mism = gi != det["idx"]
        r["coords_checked"] += int(gi.size)
        r["boundary_mismatches"] += int(mism.sum())
        if mism.any():
            t = O.format_boundaries(O.format_levels(bits))
            dist = np.min(np.abs(det["z"][mism][:, None] - t[None, :]), axis=1)
            r["mismatches_outside_band"] += int((dist >= 1e-5).sum())
        ref = det["norm64"]
        ok = ref > 0
        rel = np.abs(gn.astype(np.float64)[ok] - ref[ok]) / ref[ok]
        r["max_norm_rel_err"] = max(r["max_norm_rel_err"], float(rel.max()) if rel.size else 0.0)
        ulp = np.abs(_ordered_f16(gx) - _ordered_f16(O.decode(gp, gn, bits, 42, D)))
        r["max_decode_ulp"] = max(r["max_decode_ulp"], int(ulp.max()))

    def summary(self):
        tot = sum(v["coords_checked"] for v in self.t.values())
        mis = sum(v["boundary_mismatches"] for v in self.t.values())
        return {"coords_checked": tot, "boundary_mismatches": mis,
                "boundary_mismatch_frac": mis / tot if tot else None,
                "mismatches_outside_band": sum(v["mismatches_outside_band"] for v in self.t.values()),
                "max_norm_rel_err": max((v["max_norm_rel_err"] for v in self.t.values()), default=None),
                "max_decode_ulp": max((v["max_decode_ulp"] for v in self.t.values()), default=None),
                "per_tensor": self.t}


def _gpu_sample(K, torch, S, rows, seed=0):
    """`rows` random rows of the benchmarked K and V tensors and the GPU's
    codes, norms and decoded rows for them at 2, 3 and 4 bits: the codes and
    norms the timed step's encodes left in its buffers, the decode re-run
    on them with the step's own launch (one bulk tq_decode per tensor)."""
    n = S["n"]
    idx = torch.randperm(n, generator=torch.Generator().manual_seed(seed))[:rows].sort().values.cuda()
    xs = {t: S["xs"][t][idx].cpu().numpy() for t in "KV"}
    gpu = {}
    for b in BITS:
        for t in "KV":
            K.tq_decode(S["codecs"][b].ctx, S["packed"][b, t], S["norms"][b, t], n, S["out"])
            gpu[b, t] = (S["packed"][b, t][idx].cpu().numpy(), S["norms"][b, t][idx].cpu().numpy(),
                         S["out"][idx].cpu().numpy())
    torch.cuda.synchronize()
    return xs, gpu


def _timed_oracle_chunks(xk, xv, seconds, start, chunk, tally=None, gpu=None):
    """Oracle steps on consecutive chunks of the sample from row `start` until
    about `seconds` of oracle time; returns (rows done, bytes, seconds). The
    comparison with the GPU's outputs (when given) is not timed."""
    import oracle as O

    t_total, done, nbytes = 0.0, 0, 0
    while t_total < seconds and start + done + chunk <= len(xk):
        r0, r1 = start + done, start + done + chunk
        for bits in BITS:
            for name, xs in (("K", xk), ("V", xv)):
                t0 = time.perf_counter()
                det = O.encode_detail(xs[r0:r1], bits, 42)
                O.decode(det["packed"], det["norms"], bits, 42, D)
                t_total += time.perf_counter() - t0
                nbytes += 2 * (2 * D) * chunk
                if tally is not None:
                    gp, gn, gx = gpu[bits, name]
                    tally.add(bits, name, det, gp[r0:r1], gn[r0:r1], gx[r0:r1])
        done += chunk
    return done, nbytes, t_total


def _cpu_baseline(xk, xv, gpu=None, seconds_target=9.0, single_thread_seconds=3.0, chunk=2048):
    """The fp64 oracle, as it stands, on a bounded sample of the same
    workload: the benchmarked step (K and V, encode + decode at 2, 3 and 4
    bits) on chunks of the sampled rows, first with numpy's thread pool on
    every core for about `seconds_target`, then on one thread for about
    `single_thread_seconds`. With the GPU's outputs for the same rows, every
    processed row is also compared with the oracle (untimed)."""
    tally = _ParityTally() if gpu is not None else None
    cores = _oracle_cores()
    done, nbytes, t_all = _timed_oracle_chunks(xk, xv, seconds_target, 0, chunk, tally, gpu)
    single = None
    try:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            d1, b1, t1 = _timed_oracle_chunks(xk, xv, single_thread_seconds, done, chunk // 4)
        if d1:
            single = {"value": b1 / t1 / 1e9, "unit": "GB/s", "cores": 1,
                      "sample": f"{d1} further rows of each tensor ({t1:.1f} s)"}
    except ImportError:
        pass
    out = {"value": nbytes / t_all / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": f"{done} random rows of each of the layer's K and V tensors, encode+decode at 2, 3 and 4 "
                     f"bits, fp64 numpy on {cores} threads ({t_all:.1f} s)",
           "single_thread": single}
    return out, (tally.summary() if tally is not None else None)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import kv_cache_vector_turboquant_b200 as K
    import tq_workloads as W

    torch.cuda.set_device(local_rank)
    S = _codec_step_setup(K, W, torch, rank)
    launches = S["launches"]
    fp16eq_step = sum(L[4] for L in launches)

    def step(evs=None):
        for i, L in enumerate(launches):
            if evs is not None:
                evs[i][0].record()
            L[2]()
            if evs is not None:
                evs[i][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    err = K.tq_device_error()
    evs = [[(_ev(torch), _ev(torch)) for _ in launches] for _ in range(args.steps)]
    t0, t1 = _ev(torch), _ev(torch)
    with ClockSampler(local_rank) as clk:
        # keep the GPU under the same load for ~1 s so the sampler (200 ms
        # period) records clocks under load, then time exactly `steps` steps
        settle0 = time.perf_counter()
        while time.perf_counter() - settle0 < 1.0:
            step()
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record()
        for s in range(args.steps):
            step()
        t1.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = reduce_max_ms(t0.elapsed_time(t1), world, dist, "cuda")
        # per-launch durations from a second loop of the same `steps` steps with
        # an event pair around every launch: events between launches serialise
        # them (about 2.7 us per launch measured), so the headline loop above
        # has only its two bracketing events
        torch.cuda.synchronize()
        for s in range(args.steps):
            step(evs[s])
        torch.cuda.synchronize()
    ms_step = ms / args.steps

    # per-kernel averages (second loop)
    per = {}
    for s in range(args.steps):
        for i, L in enumerate(launches):
            per.setdefault((L[0], L[1]), []).append((evs[s][i][0].elapsed_time(evs[s][i][1]), L[3]))
    peak, peak_kind = _peaks()
    kernels = {}
    for (kind, b), vals in per.items():
        avg = statistics.mean(v[0] for v in vals) / 1e3
        kernels[f"{kind}_b{b}"] = {"us": avg * 1e6, "us_median": statistics.median(v[0] for v in vals) * 1e3,
                                   "us_best": min(v[0] for v in vals) * 1e3, "GBps": vals[0][1] / avg / 1e9,
                                   "frac": vals[0][1] / avg / 1e9 / peak,
                                   "frac_of_nominal": vals[0][1] / avg / 1e9 / HBM_NOMINAL_GBS,
                                   "share": sum(v[0] for v in vals)}
    tot = sum(v["share"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["share"] / tot
    # each launch of the step also timed back to back (`steps` calls between
    # two events): the event pair around every launch above adds ~2-3 us each
    for kind, b, fn, alg, _ in launches:
        t = _bracketed_ms(torch, fn, args.steps) / 1e3
        k = kernels[f"{kind}_b{b}"]
        k["us_b2b"] = t * 1e6
        k["GBps_b2b"] = alg / t / 1e9
        k["frac_b2b"] = alg / t / 1e9 / peak
    dom_name = max(kernels, key=lambda n: kernels[n]["share"])
    dom = kernels[dom_name]
    src = "tq_encode_tc.cu" if dom_name.startswith("encode") else "tq_decode_tc.cu"
    traffic = _profile_traffic(src, f"{dom_name.split('_')[0]}_llama_layer_{dom_name.split('_')[1]}.txt")
    # the dominant kernel's average launch duration: its launches of the step
    # (the K and V tensors, each larger than L2) back to back, `steps` times,
    # between two events
    dom_calls = [L[2] for L in launches if f"{L[0]}_b{L[1]}" == dom_name]

    def dom_round():
        for f in dom_calls:
            f()

    dom_s = _bracketed_ms(torch, dom_round, args.steps) / len(dom_calls) / 1e3
    alg_dom = per[tuple([dom_name.split('_')[0], int(dom_name[-1])])][0][1]
    roof = {"bound": "hbm", "kernel": dom_name, "achieved": alg_dom / dom_s / 1e9, "peak": peak, "unit": "GB/s",
            "frac": alg_dom / dom_s / 1e9 / peak, "traffic": traffic,
            "peak_kind": f"{peak_kind} copy (MEASURED_PEAKS.json hbm_gbs)",
            "algorithmic_bytes_per_launch": alg_dom, "launch_us": dom_s * 1e6,
            "frac_of_nominal": alg_dom / dom_s / 1e9 / HBM_NOMINAL_GBS, "nominal_gbs": HBM_NOMINAL_GBS,
            "launch_us_with_events": dom["us"],
            "timing": "the kernel's launches (one per step, K and V together) back to back between two CUDA events"}

    result = {
        "metric": "encode/decode GB/s (fp16-equivalent) & % of HBM roofline; fused attn tokens/s",
        "value": job_throughput(fp16eq_step, args.steps, world, ms),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": LLAMA_WORKLOAD, "head_dim": D, "vectors_per_tensor": S["n"],
                   "vectors_per_launch": 2 * S["n"],
                   "l2": "inputs larger than L2 (256 MiB of fp16 per launch; no launch re-reads what the previous "
                         "wrote)",
                   "parallelism": f"replicas x{world} (one layer per rank, no collective)"},
        "roofline": roof,
        "kernels": kernels,
        "clocks": clk.summary(),
        "gpu_launches": len(launches) * args.steps,
        "kernel_timing": "per-launch CUDA events in a second loop of the same steps right after the timed one "
                         "(events between launches add ~2.7 us each, so the timed loop has none)",
        "device_error_after_warmup": list(err),
    }
    # end to end through the public API with pinned host buffers
    # 8 steps: the fill and drain of the chunk pipeline (one chunk's round
    # trip) amortised over more of the run (3 steps: 74.0, 8 steps: 75.1 GB/s)
    result["e2e"] = _e2e(K, torch, S, max(2, min(args.steps, 8)), world, dist)
    if not args.skip_extras:
        result["attn"] = _bench_attention(K, W, torch, max(args.steps, 5), max(args.warmup, 3),
                                          float(result["clocks"].get("sm_mhz") or 1965.0))
        at = result["attn"]
        result["attn_summary"] = {"tokens_per_s": at["tokens_per_s"], "us_per_step": at["ms_per_step"] * 1e3,
                                  "GBps": at["roofline"]["achieved"], "frac": at["roofline"]["frac"],
                                  "paged_us_per_step": at["paged"]["ms_per_step"] * 1e3,
                                  "paged_frac": at["paged"]["frac"]}
        result["append"] = _bench_append(K, W, torch)
        result["long_context"] = _bench_long_context(K, W, torch)
        result["offset_variant"] = _bench_offset_variant(K, W, torch)
    if rank == 0 and world == 1 and not args.skip_cpu:
        xs, gpu = _gpu_sample(K, torch, S, 131072)
        result["cpu_baseline"], result["parity"] = _cpu_baseline(xs["K"], xs["V"], gpu)
    result["native_libs_loaded"] = _loaded_native_libs()
    return _front(result)


# keys printed first, so that a reader (or a tool that keeps only the head of
# the line) sees the headline, the roofline, the parity tally and the
# attention figures before the detail
_FRONT = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
          "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "clocks", "gpu_launches", "parity",
          "attn_summary", "cpu_baseline"]


def _front(result: dict) -> dict:
    out = {k: result[k] for k in _FRONT if k in result}
    out.update({k: v for k, v in result.items() if k not in out})
    return out


def _e2e(K, torch, S, steps, world, dist, chunk_rows=131072, n_streams=8):
    """End to end through the public API: every step copies each tensor's
    fp16 rows from pinned host memory, encodes, copies codes and norms back,
    copies them to the device again, decodes and copies the fp16 rows back,
    at 2, 3 and 4 bits. Each tensor is streamed in chunks of `chunk_rows`
    rows (one tq_encode / tq_decode call per chunk on its own slices of the
    device buffers), the chunks dealt round-robin to `n_streams` streams, so
    host-to-device copies, kernels and device-to-host copies of different
    chunks overlap."""
    n = S["n"]
    host_x = {t: S["xs"][t].cpu().pin_memory() for t in "KV"}
    host_p = {k: v.cpu().pin_memory() for k, v in S["packed"].items()}
    host_n = {k: v.cpu().pin_memory() for k, v in S["norms"].items()}
    host_o = {t: torch.empty(n, D, dtype=torch.float16).pin_memory() for t in "KV"}
    dx = {t: torch.empty(n, D, dtype=torch.float16, device="cuda") for t in "KV"}
    dp = {(b, t): torch.empty(n, S["codecs"][b].packed_bytes, dtype=torch.uint8, device="cuda")
          for b in BITS for t in "KV"}
    dn = {t: torch.empty(n, dtype=torch.float32, device="cuda") for t in "KV"}
    streams = [torch.cuda.Stream() for _ in range(n_streams)]
    items = [(t, r0, min(n, r0 + chunk_rows)) for r0 in range(0, n, chunk_rows) for t in "KV"]
    h2d = d2h = 0

    def step():
        for b in BITS:
            c = S["codecs"][b].ctx
            for i, (t, r0, r1) in enumerate(items):
                m = r1 - r0
                x, p, nr = dx[t][r0:r1], dp[b, t][r0:r1], dn[t][r0:r1]
                hp, hn = host_p[b, t][r0:r1], host_n[b, t][r0:r1]
                with torch.cuda.stream(streams[i % n_streams]):
                    x.copy_(host_x[t][r0:r1], non_blocking=True)  # encode: rows in, codes and norms out
                    K.tq_encode(c, x, m, p, nr)
                    hp.copy_(p, non_blocking=True)
                    hn.copy_(nr, non_blocking=True)
                    p.copy_(hp, non_blocking=True)  # decode: codes and norms in, rows out
                    nr.copy_(hn, non_blocking=True)
                    K.tq_decode(c, p, nr, m, x)
                    host_o[t][r0:r1].copy_(x, non_blocking=True)

    def run(k):
        ev0 = _ev(torch)
        ev0.record()
        for st in streams:
            st.wait_event(ev0)
        for _ in range(k):
            step()
        for st in streams:
            torch.cuda.current_stream().wait_stream(st)

    run(1)
    torch.cuda.synchronize()
    e0, e1 = _ev(torch), _ev(torch)
    if world > 1:
        dist.barrier()
    e0.record()
    run(steps)
    e1.record()
    torch.cuda.synchronize()
    ms = reduce_max_ms(e0.elapsed_time(e1), world, dist, "cuda")
    for b in BITS:
        P = S["codecs"][b].packed_bytes
        h2d += 2 * (n * 2 * D) + 2 * (n * P + n * 4)
        d2h += 2 * (n * P + n * 4) + 2 * (n * 2 * D)
    fp16eq = 12 * 2 * D * n
    return {"value": job_throughput(fp16eq, steps, world, ms), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "note": f"tq_encode/tq_decode with inputs copied from pinned host memory and results copied back; "
                    f"each tensor in chunks of {chunk_rows} rows dealt round-robin to {n_streams} streams "
                    f"(copies in both directions and kernels of different chunks overlap)"}


def run_reference(args):
    """The fp64 oracle on the host cores, as it stands: each step is the
    benchmarked step (K and V, encode + decode at 2, 3 and 4 bits) on a fixed
    sample of rows, sized so the whole run ends within a few minutes."""
    rows = 2048
    xk, xv = _oracle_sample(rows, 1)
    for _ in range(args.warmup):
        _oracle_step(xk, xv)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += _oracle_step(xk, xv)
    dt = time.perf_counter() - t0
    val = nbytes / dt / 1e9
    sample = (f"{rows} random rows of each of the layer's K and V tensors per step, encode+decode at 2, 3 and 4 "
              f"bits, fp64 numpy on {_oracle_cores()} threads")
    return {"impl": "reference", "metric": "encode/decode GB/s (fp16-equivalent) & % of HBM roofline; "
                                           "fused attn tokens/s",
            "value": val, "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": LLAMA_WORKLOAD, "head_dim": D, "vectors_per_tensor": 8 * 8192 * 8,
                       "sample": sample},
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": _oracle_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "native_libs_loaded": _loaded_native_libs()}


PROFILE_CASES = ["encode_b2", "encode_b3", "encode_b4", "decode_b2", "decode_b3", "decode_b4", "attn"]


def run_sustained(seconds: float = 2.5):
    """Each codec launch of the benchmarked step alone (the layer's K and V in
    one call, tensor-core kernels), the decode-step attention alone and the
    whole 6-launch step, each run back to back for `seconds` so the GPU
    reaches its power limit; then 50 timed launches (steps). nvidia-smi is
    sampled over the second half of each phase: the median SM clock and
    board power there say which work sets the clock under the power limit."""
    import torch

    import kv_cache_vector_turboquant_b200 as K
    import tq_workloads as W

    torch.cuda.set_device(0)
    S = _codec_step_setup(K, W, torch, 0)
    phases = [(f"{kind}_b{b}", fn) for kind, b, fn, _, _ in S["launches"]]
    phases.append(("codec_step", lambda: [L[2]() for L in S["launches"]]))
    a = ATTN
    q, k, v = W.decode_step(a["B"], a["Hq"], a["Hkv"], a["S"], a["d"])
    kc, vc = K.TurboQuant(a["d"], a["kb"]), K.TurboQuant(a["d"], a["vb"])
    kp, kn = kc.encode(k)
    vp, vn = vc.encode(v)
    del k, v
    pos = torch.full((a["B"],), a["S"], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(K.tq_attend_workspace_bytes(a["B"], a["Hq"], a["d"], a["S"]), dtype=torch.uint8, device="cuda")
    phases.append(("attention_step", lambda: K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos, out=out, workspace=ws)))
    res = []
    for name, fn in phases:
        t0 = time.time()
        while time.time() - t0 < seconds / 2:
            for _ in range(20):
                fn()
            torch.cuda.synchronize()
        with ClockSampler(torch.cuda.current_device(), with_power=True) as cs:
            while time.time() - t0 < seconds:
                for _ in range(20):
                    fn()
                torch.cuda.synchronize()
            e0, e1 = _ev(torch), _ev(torch)
            e0.record()
            for _ in range(50):
                fn()
            e1.record()
            torch.cuda.synchronize()
        res.append({"phase": name, "us": e0.elapsed_time(e1) / 50 * 1e3, **cs.summary()})
    st = K.tq_device_error()
    return {"sustained": res, "seconds_per_phase": seconds, "device_error": list(st),
            "note": "each phase alone, back to back; clock and power are nvidia-smi medians over its second half"}


def run_profile_case(case: str, launches: int = 3):
    """A small, self-contained case for Nsight Compute: a few launches of one
    kernel on the benchmark's shapes (the layer's K and V, 256 MiB of fp16,
    larger than L2; the decode-step cache is ~0.4 GB), after one warm-up
    launch."""
    import torch

    import kv_cache_vector_turboquant_b200 as K
    import tq_workloads as W

    torch.cuda.set_device(0)
    if case == "attn":
        a = ATTN
        q, k, v = W.decode_step(a["B"], a["Hq"], a["Hkv"], a["S"], a["d"])
        kc, vc = K.TurboQuant(a["d"], a["kb"]), K.TurboQuant(a["d"], a["vb"])
        kp, kn = kc.encode(k)
        vp, vn = vc.encode(v)
        del k, v
        pos = torch.full((a["B"],), a["S"], dtype=torch.int32, device="cuda")
        for _ in range(1 + launches):
            K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos)
    else:  # the benchmarked launch: the layer's K and V in one [2 n, D] buffer
        kind, b = case.split("_b")
        b = int(b)
        k, v = W.llama_layer(device="cuda")
        x = torch.cat([k.reshape(-1, D), v.reshape(-1, D)])
        del k, v
        c = K.TurboQuant(D, b)
        p, n = c.encode(x)
        out = torch.empty_like(x)
        for _ in range(1 + launches):
            if kind == "encode":
                c.encode(x, out=(p, n))
            else:
                c.decode(p, n, out=out)
    torch.cuda.synchronize()
    st = K.tq_device_error()
    print(json.dumps({"profile_case": case, "launches": 1 + launches, "device_error": list(st)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile", choices=PROFILE_CASES, default=None,
                    help="run a few launches of one kernel for Nsight Compute and exit")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-extras", action="store_true", help="skip the attention and append loops")
    ap.add_argument("--skip-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--sustained", action="store_true",
                    help="time each codec launch, the codec step and the attention step alone at the power limit "
                         "(with clock and power) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.sustained:
        print(json.dumps(run_sustained()), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    import torch.distributed as dist

    if world > 1:
        from datetime import timedelta

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
