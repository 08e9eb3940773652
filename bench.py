#!/usr/bin/env python
"""Benchmark of the compressed-weight hot path on B200.

One step = the whole hot path over one batch of synthetic input on the
Llama-3.1-8B gate_proj shape (W 14336x4096 BF16 ~ N(0, 0.02), X Mx4096 ~ N(0, 1)):
for each M in {1, 16, 64}, all four pipelines through the public C ABI
(uw_gemm):

  full            Huffman decode to BF16 in HBM -> plain tcgen05 GEMM
  exp             exponent-only decode -> reconstructive GEMM
  palette_rt      transcode to 4-bit palette indices -> reconstructive GEMM
  palette_direct  reconstructive GEMM on indices transcoded at load

Four independently drawn weight matrices (seeds 10, 12, 14, 16) are used in
rotation, one per pipeline run, so every kernel reads weights that are not in
the 126 MB L2 (each set is ~150 MB compressed + its workspace traffic).

``value`` = algorithmic bytes of the whole step (sum over its kernels of the
bytes each must move: compressed streams read, preprocessed weights written and
read back, X read, Y written) / device time of the step, in GB/s, summed over
ranks.  The timed region runs untraced.  A second, traced pass of the same
steps (the library's own CUDA events around each launch, uw_trace_enable)
attributes time to kernels; those per-launch times include each launch's own
start-up and event cost (about 6 us on this part).  The roofline's launch time
is measured apart: the dominant kernel alone, launched back to back over the
same M mix and weight rotation, between two events on its stream.

Multi-GPU: replicas only (the path does not shard; each rank runs the same
independent step), timing is the max over ranks.

``--impl reference`` times the CPU oracle (test infrastructure, bit-by-bit
canonical Huffman decode + FP64 matmul) on a bounded sample of the same
workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Huffman decode GB/s; fused decompress-GEMM TFLOP/s & µs vs BF16 GEMM, M=1..1024"
WORKLOAD = "gate_14336x4096"
MS = (1, 16, 64)
PIPES = ("full", "exp", "palette_rt", "palette_direct")
N_SETS = 4
REF_ROWS = 48             # oracle rows per reference-arm step (~2 s of CPU work)
CPU_BASELINE_ROWS = 300   # oracle rows for the cpu_baseline leg (~12 s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 7700.0  # B200 HBM3e, nominal (HGX)

# DRAM traffic per launch from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum of one launch), valid only while the kernel source
# (src_sha, see _kernel_src_sha) is unchanged.
TRAFFIC = {
    "gemm_palette": {"bytes_per_launch": 89.744128e6 + 2.605312e6, "src_sha": "0bd3631b51fba772",
                     "capture": "palette GEMM, 14336x4096, M = 1 launch"},
    "decode_full": {"bytes_per_launch": 87.415040e6 + 64.024064e6, "src_sha": "2a78f2d845afbc82",
                    "capture": "full decode, 14336x4096 (output partly still in L2)"},
}

def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-large-m", action="store_true",
                    help="skip the large-M matmul block (gate M = 1024, down M = 256, 1024) "
                         "and the Huffman-direct block (pipeline 5, M = 1, 2, 8)")
    # single-kernel runs for profilers: three launches of one kernel, nothing timed
    ap.add_argument("--only", choices=("decode_full", "decode_exp", "transcode", "gemm_bf16",
                                       "gemm_exp", "gemm_palette", "gemv_bf16", "gemv_exp",
                                       "gemv_palette", "decode_dot"))
    ap.add_argument("--m", type=int, default=1, help="tokens for --only gemm_*, gemv_*, decode_dot")
    # the Llama-3.1-8B-shaped MLP stack end to end (prints its own JSON line)
    ap.add_argument("--mlp-layers", type=int, default=0,
                    help="time uw_mlp_forward over this many gate/up/down layers")
    ap.add_argument("--mlp-ms", default="1,64,256,1024")
    ap.add_argument("--mlp-force-down", default="",
                    help="comma list of pipelines (2, 3, or 5 at M <= 8) to force on every "
                         "down_proj, gate/up on pipeline 4: times the stack with the preprocessing "
                         "overlap off, "
                         "on, and with the tuned decoder/GEMM SM split")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------- algorithmic bytes --

def _alg_bytes(kind, st, M, N, K, x_frac=1.0):
    """Bytes a kernel launch must move at minimum: compressed streams read,
    preprocessed weights written / read back, X read once (x_frac of it when
    only a slice of W's rows is processed), Y written once."""
    T = N * K
    stream = st["bytes_stream"] + st["bytes_offsets"]
    esc = st["bytes_escape"]
    xy = x_frac * 2 * M * K + 2 * M * N
    b = {
        "decode_full": stream + T + 2 * T,
        "decode_exp": stream + T,
        "transcode": stream + T // 2,
        "gemm_bf16": 2 * T + xy,
        "gemm_exp": 2 * T + xy,
        "gemm_palette": T + T // 2 + esc + xy,
        "decode_dot": stream + T + xy,
    }
    return b[kind.replace("gemv_", "gemm_")]


def _block_time(uw, torch, kind, handles, stats, X, Y, Ms, N, K, stream, rounds):
    """Device time of `rounds` x len(Ms) x len(handles) launches of one kernel,
    back to back on `stream` (one untimed round first).  Returns (ms, launches,
    algorithmic bytes), or None for a kernel the public calls cannot launch
    alone (the BF16 and exponent GEMMs always follow their decode)."""
    if kind not in ("decode_full", "decode_exp", "transcode", "gemm_palette"):
        return None

    out = None
    if kind == "decode_full":
        out = torch.empty(N * K, dtype=torch.int16, device="cuda")
    elif kind == "decode_exp":
        out = torch.empty(N * K, dtype=torch.uint8, device="cuda")
    elif kind == "transcode":
        out = torch.empty(N * K // 2, dtype=torch.uint8, device="cuda")

    def launch(h, m):
        if kind == "decode_full":
            uw.uw_decode_full(h, out)
        elif kind == "decode_exp":
            uw.uw_decode_exp(h, out)
        elif kind == "transcode":
            uw.uw_transcode_palette(h, out)
        elif kind == "gemm_palette":
            uw.uw_gemm(h, X[m], Y[(m, "palette_direct")], m, uw.PIPELINES["palette_direct"])

    def one_round():
        b = 0
        for m in (Ms if kind.startswith(("gemm", "gemv")) else Ms[:1]):
            for i, h in enumerate(handles):
                launch(h, m)
                b += _alg_bytes(kind, stats[i], m, N, K)
        return b

    one_round()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    total = 0
    for _ in range(rounds):
        total += one_round()
    e1.record(stream)
    torch.cuda.synchronize()
    n = rounds * (len(Ms) if kind.startswith(("gemm", "gemv")) else 1) * len(handles)
    return e0.elapsed_time(e1), n, total


# Large-M matmul block of the bench line: (workload, M) pairs, and the
# weight sets rotated per call so a pipeline's weights are not in L2.
LARGE_M = (("gate_14336x4096", 1024), ("down_4096x14336", 256), ("down_4096x14336", 1024))
LARGE_M_SETS = 2


def _large_m_block(uw, torch, stream, peaks, reps=8):
    """Every pipeline at the metric's large M on the gate and down shapes:
    whole-pipeline time (calls back to back between two events, weight sets
    rotated), its split into preprocessing and GEMM (the library's traced
    events), the GEMM's TFLOP/s and its roofline time max(2MNK / BF16 peak,
    algorithmic bytes / HBM peak); then the autotuner's choice for that M
    (uw_autotune over pipelines, token tiles, ring depths, CTA pairs) timed
    the same way; torch.matmul on the decoded BF16 weights for context."""
    import numpy as np
    import synthdata
    out = {}
    by_wl = {}
    for wl, M in LARGE_M:
        by_wl.setdefault(wl, []).append(M)
    for wl, Ms in by_wl.items():
        spec = synthdata.WORKLOADS[wl]
        N, K = spec["N"], spec["K"]
        hs, sts = [], []
        for i in range(LARGE_M_SETS):
            w = synthdata.normal(N, K, spec["std"], spec["seed_w"] + 2 * i)
            h = uw.uw_encode(w, stream=stream)
            hs.append(h)
            sts.append(h.stats())
            del w
        need = max(uw.uw_workspace_bytes(hs[0], uw.PIPELINES[p], m) for p in PIPES for m in Ms)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        for h in hs:
            uw.uw_set_workspace(h, ws)
        wbf = []
        for h in hs:
            t = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
            uw.uw_decode_full(h, t)
            wbf.append(t)
        for M in Ms:
            X = torch.from_numpy(synthdata.activations(M, K, spec["seed_x"] + M).view(np.int16)) \
                .cuda().view(torch.bfloat16)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            flops = 2.0 * M * N * K
            rec = {}
            for p in PIPES:
                pre, gemm = _run_kernels(p, M)
                call = lambda i: uw.uw_gemm(hs[i % LARGE_M_SETS], X, Y, M, uw.PIPELINES[p])
                for i in range(3):
                    call(i)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for i in range(reps):
                    call(i)
                e1.record(stream)
                torch.cuda.synchronize()
                total_us = 1e3 * e0.elapsed_time(e1) / reps
                # traced split (events around each kernel)
                for h in hs:
                    uw.uw_trace_read(h)
                    uw.uw_trace_enable(h, True)
                for i in range(reps):
                    call(i)
                torch.cuda.synchronize()
                tr = [x for h in hs for x in uw.uw_trace_read(h)]
                for h in hs:
                    uw.uw_trace_enable(h, False)
                g_ms = [ms for kind, ms in tr if kind == gemm]
                p_ms = [ms for kind, ms in tr if kind == pre] if pre else []
                gemm_us = 1e3 * statistics.median(g_ms)
                pre_us = 1e3 * statistics.median(p_ms) if p_ms else 0.0
                gbytes = _alg_bytes(gemm, sts[0], M, N, K)
                t_roof = max(flops / (peaks["bf16_tflops"] * 1e12), gbytes / (peaks["hbm_gbs"] * 1e9))
                rec[p] = {"total_us": total_us, "preprocess_us_traced": pre_us,
                          "gemm_us_traced": gemm_us, "gemm_tflops": flops / (gemm_us * 1e-6) / 1e12,
                          "gemm_roofline_us": 1e6 * t_roof,
                          "gemm_frac": 1e6 * t_roof / gemm_us,
                          "gemm_bound": "tensor" if flops / (peaks["bf16_tflops"] * 1e12) >=
                          gbytes / (peaks["hbm_gbs"] * 1e9) else "hbm"}
            # the autotuner's choice for this M (pipeline, token tile, ring
            # depth, CTA pairs), timed the same way
            uw.uw_autotune(hs, [M])
            choice = uw.uw_get_choice(hs[0], M)
            call = lambda i: uw.uw_gemm(hs[i % LARGE_M_SETS], X, Y, M, uw.UW_PIPE_AUTO)
            for i in range(3):
                call(i)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(reps):
                call(i)
            e1.record(stream)
            torch.cuda.synchronize()
            auto_us = 1e3 * e0.elapsed_time(e1) / reps
            rec["autotuned"] = {"total_us": auto_us, "choice": choice,
                                "tflops_whole_pipeline": flops / (auto_us * 1e-6) / 1e12}
            ts = []
            for i in range(3 + reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                torch.matmul(X, wbf[i % LARGE_M_SETS].t())
                b.record(stream)
                b.synchronize()
                if i >= 3:
                    ts.append(1e3 * a.elapsed_time(b))
            rec["torch_matmul_bf16_us"] = statistics.median(ts)
            rec["torch_matmul_bf16_tflops"] = flops / (rec["torch_matmul_bf16_us"] * 1e-6) / 1e12
            out[f"{wl}/M{M}"] = rec
        for h in hs:
            if uw.uw_last_device_status(h) != uw.UW_OK:
                raise RuntimeError("device status")
            h.free()
        del wbf, ws
    return out


# Huffman-direct product block of the bench line: shapes, token counts, and
# the weight sets rotated per call.
HDOT = (("gate_14336x4096", (1, 2, 8)), ("down_4096x14336", (1, 2, 8)))
HDOT_SETS = 2


def _hdot_block(uw, torch, stream, peaks, reps=10):
    """Pipeline 5 (the stream decoded inside the matmul, no preprocessing
    pass) at small M on the gate and down shapes: whole-call time back to back
    (weight sets rotated), the kernel's traced time, its algorithmic bytes
    (stream, offsets, S, X, Y) and fraction of HBM; beside it the whole
    pipelines 2, 3 and 4 at the same M, timed the same way."""
    import numpy as np
    import synthdata
    out = {}
    for wl, Ms in HDOT:
        spec = synthdata.WORKLOADS[wl]
        N, K = spec["N"], spec["K"]
        hs = []
        for i in range(HDOT_SETS):
            w = synthdata.normal(N, K, spec["std"], spec["seed_w"] + 2 * i)
            hs.append(uw.uw_encode(w, stream=stream))
            del w
        st = hs[0].stats()
        need = max(uw.uw_workspace_bytes(hs[0], p, m) for p in (2, 3, 5) for m in Ms)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        for h in hs:
            uw.uw_set_workspace(h, ws)
        for M in Ms:
            X = torch.from_numpy(synthdata.activations(M, K, spec["seed_x"] + M).view(np.int16)).cuda()
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

            def chain(p):
                call = lambda i: uw.uw_gemm(hs[i % HDOT_SETS], X, Y, M, p)
                for i in range(3):
                    call(i)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for i in range(reps):
                    call(i)
                e1.record(stream)
                torch.cuda.synchronize()
                return 1e3 * e0.elapsed_time(e1) / reps

            rec = {"total_us": chain(uw.UW_PIPE_HUFFMAN_DIRECT)}
            for h in hs:
                uw.uw_trace_read(h)
                uw.uw_trace_enable(h, True)
            for i in range(reps):
                uw.uw_gemm(hs[i % HDOT_SETS], X, Y, M, uw.UW_PIPE_HUFFMAN_DIRECT)
            torch.cuda.synchronize()
            tr = [ms for h in hs for kind, ms in uw.uw_trace_read(h) if kind == "decode_dot"]
            for h in hs:
                uw.uw_trace_enable(h, False)
            k_us = 1e3 * statistics.median(tr)
            alg = _alg_bytes("decode_dot", st, M, N, K)
            rec.update({"kernel_us_traced": k_us, "alg_bytes": alg,
                        "bytes_per_weight": (st["bytes_stream"] + st["bytes_offsets"] + N * K) / (N * K),
                        "frac_hbm_b2b": alg / (rec["total_us"] * 1e-6) / (peaks["hbm_gbs"] * 1e9),
                        "frac_hbm_traced": alg / (k_us * 1e-6) / (peaks["hbm_gbs"] * 1e9)})
            for p in ("exp", "palette_rt", "palette_direct"):
                rec[f"{p}_total_us"] = chain(uw.PIPELINES[p])
            out[f"{wl}/M{M}"] = rec
        for h in hs:
            if uw.uw_last_device_status(h) != uw.UW_OK:
                raise RuntimeError("device status")
            h.free()
        del ws
    return out


def _run_kernels(pipe, M):
    """(preprocessing kernel or None, matmul kernel) of a pipeline at M tokens
    with the library's default variant (the tensor-core GEMM at every M)."""
    pre = {"full": "decode_full", "exp": "decode_exp", "palette_rt": "transcode",
           "palette_direct": None}[pipe]
    gemm = {"full": "bf16", "exp": "exp"}.get(pipe, "palette")
    return pre, "gemm_" + gemm


# ------------------------------------------------------------------- clocks --

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        busy = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- CPU oracle --

def cpu_oracle_sample(rows=4, ms=MS, target_s=None):
    """Oracle on a bounded sample of the workload: the first ``rows`` rows of the
    weight matrix as a matrix of their own, all four pipelines (bit-by-bit
    decode / transcode, FP64 matmul) for every M.  Returns (GB/s, seconds,
    description).  Single thread (BLAS limited to 1)."""
    import numpy as np
    import oracle
    import synthdata
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        limiter = None
    w = synthdata.workload(WORKLOAD, rows=rows)
    n, k = w.shape
    enc = oracle.encode(w, chunk_syms=256)
    st = {"bytes_stream": (enc.total_bits + 7) // 8, "bytes_offsets": enc.offsets.size * 4,
          "bytes_escape": enc.esc_exp.size + enc.esc_bits.size * 4 + enc.esc_off.size * 4}
    xs = {m: synthdata.activation_for(WORKLOAD, m) for m in ms}
    alg = 0
    t0 = time.perf_counter()
    for m in ms:
        x = xs[m]
        for pipe in PIPES:
            if pipe == "full":
                wd = oracle.decode_full(enc)
            elif pipe == "exp":
                wd = oracle.join_fields(enc.sm, oracle.decode_exp(enc))
            elif pipe == "palette_rt":
                from oracle.container import rebuild_from_palette
                wd = rebuild_from_palette(enc, oracle.transcode_from_stream(enc))
            else:
                from oracle.container import rebuild_from_palette
                packed = oracle.pack_nibbles(oracle.transcode(oracle.exponent_bytes(w),
                                                              enc.palette, enc.esc))
                wd = rebuild_from_palette(enc, packed)
            y = oracle.gemm_fp64(x, wd)
            assert y.shape == (m, n)
            pre, gemm = _run_kernels(pipe, m)
            frac = n / synthdata.WORKLOADS[WORKLOAD]["N"]  # this slice's share of X traffic
            if pre:
                alg += _alg_bytes(pre, st, m, n, k, frac)
            alg += _alg_bytes(gemm, st, m, n, k, frac)
    dt = time.perf_counter() - t0
    if limiter is not None:
        limiter.unregister()
    desc = (f"first {rows} rows of {WORKLOAD} ({rows * k} weights) encoded on their own; "
            f"4 pipelines x M in {list(ms)}; oracle bit-by-bit decode + FP64 matmul, 1 thread")
    return alg / dt / 1e9, dt, desc


def _oracle_decode_range(args):
    """Worker of the all-cores CPU leg: the oracle's bit-by-bit decode of the
    chunks [c0, c1) of one encoded sample (module-level so a spawned process
    can run it)."""
    import numpy as np
    import oracle
    words, offsets, lengths, total, cs, c0, c1 = args
    words = [int(x) for x in words]  # one conversion per job, as decode_bitstream does
    out = []
    for c in range(c0, c1):
        n = min(cs, total - c * cs)
        syms, _ = oracle.decode_chunk(words, int(offsets[c]), n, lengths)
        out.append(np.asarray(syms, dtype=np.uint8))
    return c0, out


def cpu_oracle_sample_all_cores(rows=CPU_BASELINE_ROWS, ms=MS):
    """The same sample and work as cpu_oracle_sample on every host core: each
    pipeline's bit-by-bit decode split into chunk ranges over a spawned
    process pool (chunks decode independently by construction), the FP64
    matmul with BLAS on all threads.  Returns (GB/s, seconds, cores)."""
    import multiprocessing as mp
    import numpy as np
    import oracle
    import synthdata
    from oracle.container import rebuild_from_palette
    cores = os.cpu_count() or 1
    w = synthdata.workload(WORKLOAD, rows=rows)
    n, k = w.shape
    enc = oracle.encode(w, chunk_syms=256)
    st = {"bytes_stream": (enc.total_bits + 7) // 8, "bytes_offsets": enc.offsets.size * 4,
          "bytes_escape": enc.esc_exp.size + enc.esc_bits.size * 4 + enc.esc_off.size * 4}
    xs = {m: synthdata.activation_for(WORKLOAD, m) for m in ms}
    n_chunks = enc.offsets.size - 1
    step = -(-n_chunks // cores)
    jobs = []
    for c0 in range(0, n_chunks, step):
        c1 = min(c0 + step, n_chunks)
        # each job gets only its stretch of the stream, offsets rebased to it
        w0 = int(enc.offsets[c0]) // 32
        w1 = min(int(enc.offsets[c1]) // 32 + 2, enc.words.size)
        offs = enc.offsets.astype(np.int64) - 32 * w0
        jobs.append((enc.words[w0:w1].copy(), offs[:c1 + 1], enc.lengths, n * k,
                     enc.chunk_syms, c0, c1))
    ctx = mp.get_context("spawn")
    with ctx.Pool(min(cores, len(jobs))) as pool:
        pool.map(_oracle_decode_range, jobs[:1])  # workers up and importing before timing

        def decode_exp():
            parts = sorted(pool.map(_oracle_decode_range, jobs), key=lambda t: t[0])
            return np.concatenate([np.concatenate(p[1]) for p in parts]).reshape(n, k)

        alg = 0
        t0 = time.perf_counter()
        for m in ms:
            x = xs[m]
            for pipe in PIPES:
                if pipe == "full":
                    wd = oracle.join_fields(enc.sm, decode_exp())
                elif pipe == "exp":
                    wd = oracle.join_fields(enc.sm, decode_exp())
                elif pipe == "palette_rt":
                    e = decode_exp()
                    wd = rebuild_from_palette(enc, oracle.pack_nibbles(
                        oracle.transcode(e, enc.palette, enc.esc)))
                else:
                    packed = oracle.pack_nibbles(oracle.transcode(oracle.exponent_bytes(w),
                                                                  enc.palette, enc.esc))
                    wd = rebuild_from_palette(enc, packed)
                y = oracle.gemm_fp64(x, wd)
                assert y.shape == (m, n)
                pre, gemm = _run_kernels(pipe, m)
                frac = n / synthdata.WORKLOADS[WORKLOAD]["N"]
                if pre:
                    alg += _alg_bytes(pre, st, m, n, k, frac)
                alg += _alg_bytes(gemm, st, m, n, k, frac)
        dt = time.perf_counter() - t0
    return alg / dt / 1e9, dt, cores


def max_over_ranks(x, world, device="cuda"):
    """The largest of every rank's x (each rank's device time of the same timed
    steps): the job's time is its slowest replica's."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(bytes_per_rank, max_ms, world):
    """Whole-job throughput in GB/s: every replica processes bytes_per_rank in
    the timed region, which lasts max_ms (the slowest rank's time)."""
    return bytes_per_rank * world / (max_ms * 1e-3) / 1e9


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(max(args.warmup, 0)):
        cpu_oracle_sample(rows=REF_ROWS)
    vals, secs = [], []
    desc = ""
    for _ in range(args.steps):
        v, dt, desc = cpu_oracle_sample(rows=REF_ROWS)
        vals.append(v)
        secs.append(dt)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8+f64", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD} sample", "Ms": list(MS), "pipelines": list(PIPES)},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- our arm ----

def _load_build():
    import importlib.util
    spec = importlib.util.spec_from_file_location("uw_build", os.path.join(ROOT, "decode_gemm_b200",
                                                                            "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


# The sources each kernel is built from (a capture's counters stay valid while
# they are unchanged).
KERNEL_SOURCES = {
    "decode": ("decode.cu", "bf16_fields.cuh", "pdl.cuh"),
    "gemm": ("gemm.cu", "gemm_sm100.cuh", "bf16_fields.cuh", "pdl.cuh"),
    "gemv": ("gemv.cu", "bf16_fields.cuh", "pdl.cuh"),
}


def _code_only(text):
    """C++ source without comments and blank space: what the compiler sees."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def _kernel_src_sha(kind=None):
    """Digest of the code (comments and layout aside) of one kernel family's
    sources ("decode" or "gemm"), or of both."""
    files = KERNEL_SOURCES[kind] if kind else sorted(set(sum(KERNEL_SOURCES.values(), ())))
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "decode_gemm_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    _load_build().build()
    import decode_gemm_b200 as uw
    import synthdata

    wl = synthdata.WORKLOADS[args.workload]
    N, K = wl["N"], wl["K"]
    Ms = tuple(wl["Ms"]) if args.workload != WORKLOAD else MS
    stream = torch.cuda.current_stream()

    # weights: N_SETS independent draws of the same shape, encoded and resident
    handles, stats = [], []
    for i in range(N_SETS):
        if wl["kind"] == "normal":
            w = synthdata.normal(N, K, wl["std"], wl["seed_w"] + 2 * i)
        else:
            w = synthdata.student_t(N, K, wl["nu"], wl["std"], wl["seed_w"] + 2 * i)
        h = uw.uw_encode(w, stream=stream)
        handles.append(h)
        stats.append(h.stats())
        del w
    need = max(uw.uw_workspace_bytes(handles[0], uw.PIPELINES[p], m) for p in PIPES for m in Ms)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    for h in handles:
        uw.uw_set_workspace(h, ws)
    X = {m: torch.from_numpy(synthdata.activations(m, K, wl["seed_x"] + m).view(np.int16))
         .cuda().view(torch.bfloat16) for m in Ms}
    Y = {(m, p): torch.empty((m, N), dtype=torch.bfloat16, device="cuda") for m in Ms for p in PIPES}
    runs = [(m, p) for m in Ms for p in PIPES]

    def step(run0):
        for j, (m, p) in enumerate(runs):
            h = handles[(run0 + j) % N_SETS]
            uw.uw_gemm(h, X[m], Y[(m, p)], m, uw.PIPELINES[p])
        return run0 + len(runs)

    # algorithmic bytes of one step (depends only on the rotation position)
    def step_bytes(run0):
        tot = 0
        for j, (m, p) in enumerate(runs):
            st = stats[(run0 + j) % N_SETS]
            pre, gemm = _run_kernels(p, m)
            if pre:
                tot += _alg_bytes(pre, st, m, N, K)
            tot += _alg_bytes(gemm, st, m, N, K)
        return tot

    run0 = 0
    for _ in range(args.warmup):
        run0 = step(run0)
    torch.cuda.synchronize()

    # ---- device-resident timed region (untraced)
    total_bytes = sum(step_bytes(run0 + s * len(runs)) for s in range(args.steps))
    launches = args.steps * sum(1 + (_run_kernels(p, m)[0] is not None) for (m, p) in runs)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            run0 = step(run0)
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    for h in handles:
        st = uw.uw_last_device_status(h)
        if st != uw.UW_OK:
            raise RuntimeError(f"device status {uw.uw_status_str(st)}")
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = elapsed_ms / args.steps
    value = job_rate(total_bytes, elapsed_ms, world)

    # ---- traced pass: per-kernel attribution (runs rotate over handles)
    for h in handles:
        uw.uw_trace_read(h)  # discard earlier records
        uw.uw_trace_enable(h, True)
    run_start = run0
    for _ in range(args.steps):
        run0 = step(run0)
    torch.cuda.synchronize()
    traces = [uw.uw_trace_read(h) for h in handles]
    for h in handles:
        uw.uw_trace_enable(h, False)
    traced_ms = sum(ms for tr in traces for _, ms in tr)
    per_kind = {}
    per_run = {}
    cursor = [0] * N_SETS
    for s in range(args.steps):
        for j, (m, p) in enumerate(runs):
            idx = (run_start + s * len(runs) + j) % N_SETS
            tr = traces[idx]
            pre, gemm = _run_kernels(p, m)
            st = stats[idx]
            rec = {}
            for kind in ([pre] if pre else []) + [gemm]:
                c = cursor[idx]
                if c < len(tr) and tr[c][0] == kind:
                    rec[kind] = tr[c][1]
                    cursor[idx] += 1
                    b = _alg_bytes(kind, st, m, N, K)
                    agg = per_kind.setdefault(kind, {"ms": 0.0, "n": 0, "bytes": 0, "flops": 0})
                    agg["ms"] += tr[c][1]
                    agg["n"] += 1
                    agg["bytes"] += b
                    if kind.startswith(("gemm", "gemv")):
                        agg["flops"] += 2 * m * N * K
            per_run.setdefault((m, p), []).append(rec)
    dominant = max(per_kind, key=lambda k: per_kind[k]["ms"])
    peaks, peak_src = _peaks()
    d = per_kind[dominant]
    # the dominant kernel alone, back to back: the same M mix and weight
    # rotation, no events or other kernels between launches
    blk = _block_time(uw, torch, dominant, handles, stats, X, Y, Ms, N, K, stream,
                      rounds=max(args.steps // 2, 3))
    if blk is None:  # traced per-launch times instead
        blk_ms, blk_n, blk_bytes = d["ms"], d["n"], d["bytes"]
        timing = "traced per-launch events (the kernel has no standalone public launch)"
    else:
        blk_ms, blk_n, blk_bytes = blk
        timing = (f"{blk_n} launches back to back between two events (M in {list(Ms)}, "
                  f"{N_SETS} weight sets rotated)")
    achieved = blk_bytes / (blk_ms * 1e-3) / 1e9
    traffic = TRAFFIC.get(dominant)
    fam = ("decode" if dominant.startswith("decode") or dominant == "transcode"
           else "gemv" if dominant.startswith("gemv") else "gemm")
    if traffic and traffic.get("src_sha") != _kernel_src_sha(fam):
        traffic = None
    roofline = {"kernel": dominant, "bound": "hbm", "achieved": achieved,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "traffic": traffic["bytes_per_launch"] if traffic else None,
                "algorithmic_bytes_per_launch": blk_bytes / blk_n,
                "avg_launch_us": 1e3 * blk_ms / blk_n,
                "timing": timing,
                "avg_launch_us_traced": 1e3 * d["ms"] / d["n"],
                # the same kernel timed launch by launch (events around each,
                # no overlap with its neighbours; includes each launch's own
                # start-up): the isolated figure beside the back-to-back one
                "frac_traced": (d["bytes"] / (d["ms"] * 1e-3) / 1e9) / peaks["hbm_gbs"],
                "peak_source": peak_src,
                # against the nominal HBM3e figure (HGX), for context beside the measured peak
                "frac_nominal": achieved / NOMINAL_HBM_GBS}
    kernels = {k: {"launches": v["n"], "total_ms": v["ms"], "share": v["ms"] / traced_ms,
                   "GBps": v["bytes"] / (v["ms"] * 1e-3) / 1e9 if v["ms"] > 0 else None,
                   "frac_hbm": (v["bytes"] / (v["ms"] * 1e-3) / 1e9) / peaks["hbm_gbs"]
                   if v["ms"] > 0 else None}
               for k, v in per_kind.items()}
    pipelines = {}
    for (m, p), recs in per_run.items():
        def med(kind):
            xs = [r[kind] for r in recs if kind in r]
            return 1e3 * statistics.median(xs) if xs else None
        pre, gemm = _run_kernels(p, m)
        g = med(gemm) or 0.0
        pr = med(pre) if pre else 0.0
        pipelines[f"{p}/M{m}"] = {"preprocess_us": pr, "gemm_us": g, "total_us": pr + g,
                                  "gemm_tflops": 2 * m * N * K / (g * 1e-6) / 1e12
                                  if g > 0 else None}

    # ---- each preprocessing kernel alone, back to back (the traced figures
    # above carry each launch's own event and start-up cost)
    for kind in ("decode_full", "decode_exp", "transcode"):
        if kind in kernels:
            bt = _block_time(uw, torch, kind, handles, stats, X, Y, Ms, N, K, stream,
                             rounds=max(args.steps // 2, 3))
            gbs = bt[2] / (bt[0] * 1e-3) / 1e9
            kernels[kind].update({"b2b_launches": bt[1], "b2b_us": 1e3 * bt[0] / bt[1],
                                  "b2b_GBps": gbs, "b2b_frac_hbm": gbs / peaks["hbm_gbs"],
                                  "b2b_frac_nominal": gbs / NOMINAL_HBM_GBS,
                                  # BF16 weights the launch decodes (N*K*2 bytes) per second
                                  "b2b_decoded_weight_GBps":
                                      2 * N * K / (bt[0] / bt[1] * 1e-3) / 1e9})

    # ---- BF16 torch.matmul on the same box (context only)
    wbf = []
    for h in handles:
        t = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        uw.uw_decode_full(h, t)
        wbf.append(t)
    torch.cuda.synchronize()
    tm = {}
    for m in Ms:
        ts = []
        for it in range(3 + 12):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            torch.matmul(X[m], wbf[it % N_SETS].t())
            b.record(stream)
            b.synchronize()
            if it >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
        tm[f"M{m}"] = statistics.median(ts)
    # like for like, launched back to back over the rotated weight sets: torch
    # BF16 against the pipeline-4 matmul on the compressed weights
    b2b = {}
    for m in Ms:
        def chain(fn, reps=40):
            for i in range(N_SETS):
                fn(i)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(reps):
                fn(i)
            b.record(stream)
            torch.cuda.synchronize()
            return 1e3 * a.elapsed_time(b) / reps
        b2b[f"M{m}"] = {
            "torch_matmul_bf16_us": chain(lambda i: torch.matmul(X[m], wbf[i % N_SETS].t())),
            "palette_direct_us": chain(lambda i: uw.uw_gemm(handles[i % N_SETS], X[m],
                                                            Y[(m, "palette_direct")], m,
                                                            uw.PIPELINES["palette_direct"]))}
    del wbf

    # ---- the metric's large-M matmuls (gate and down shapes)
    gemm_large = None if args.no_large_m else _large_m_block(uw, torch, stream, peaks)
    # ---- the Huffman-direct product (pipeline 5) at small M
    hdot = None if args.no_large_m else _hdot_block(uw, torch, stream, peaks)

    # ---- end to end through the public call with host buffers: every step
    # copies its X in from pinned host memory and its Y out to pinned host
    # memory.  The copies run on two copy streams (one per direction),
    # double-buffered, so step s's Y copy and step s+1's X copy overlap the
    # compute; the timed region ends when the last step's Y has reached the host.
    # a step's inputs, and its outputs, packed in one buffer each (one copy
    # per direction and step: the host enqueues 21 launches a step already)
    def packed(shapes):
        flat = torch.empty(sum(int(torch.Size(sh).numel()) for sh in shapes.values()),
                           dtype=torch.bfloat16, device="cuda")
        views, at = {}, 0
        for key, sh in shapes.items():
            n = int(torch.Size(sh).numel())
            views[key] = flat[at:at + n].view(sh)
            at += n
        return flat, views

    xshapes = {m: tuple(v.shape) for m, v in X.items()}
    yshapes = {k: tuple(v.shape) for k, v in Y.items()}
    xflat, xview = zip(*(packed(xshapes) for _ in range(2)))
    yflat, yview = zip(*(packed(yshapes) for _ in range(2)))
    for m in Ms:
        xview[0][m].copy_(X[m])
    Xh = xflat[0].cpu().pin_memory()
    Yh = [torch.empty(yflat[0].shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    h2d = Xh.numel() * 2
    d2h = Yh[0].numel() * 2
    Xb, Yb = list(xview), list(yview)
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()  # one stream per direction
    ev = lambda: torch.cuda.Event()
    x_ready, x_free, y_done, y_free = ([ev(), ev()] for _ in range(4))
    start = ev()

    def step_io(run0, Xd, Yd):
        for j, (m, p) in enumerate(runs):
            h = handles[(run0 + j) % N_SETS]
            uw.uw_gemm(h, Xd[m], Yd[(m, p)], m, uw.PIPELINES[p])
        return run0 + len(runs)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    start.record(stream)
    h2d_s.wait_event(start)
    d2h_s.wait_event(start)
    run_e = run0
    e2e_bytes = 0
    for s_i in range(args.steps):
        b = s_i % 2
        with torch.cuda.stream(h2d_s):
            if s_i >= 2:
                h2d_s.wait_event(x_free[b])  # compute two steps ago is done with Xb[b]
            xflat[b].copy_(Xh, non_blocking=True)
            x_ready[b].record(h2d_s)
        stream.wait_event(x_ready[b])
        if s_i >= 2:
            stream.wait_event(y_free[b])  # Yb[b] from two steps ago is on the host
        e2e_bytes += step_bytes(run_e)
        run_e = step_io(run_e, Xb[b], Yb[b])
        x_free[b].record(stream)
        y_done[b].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(y_done[b])
            Yh[b].copy_(yflat[b], non_blocking=True)
            y_free[b].record(d2h_s)
    for b in range(min(2, args.steps)):
        stream.wait_event(y_free[b])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_rate(e2e_bytes, e2e_ms, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v1, dt1, desc = cpu_oracle_sample(rows=CPU_BASELINE_ROWS)
        va, dta, cores = cpu_oracle_sample_all_cores(rows=CPU_BASELINE_ROWS)
        cpu = {"value": va, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": desc.replace(", 1 thread", "") + f"; on all {cores} host cores "
                         "(decode chunks over a spawned process pool, BLAS on all threads)",
               "seconds": dta, "host_cpu_count": os.cpu_count(),
               "single_core": {"value": v1, "cores": 1, "seconds": dt1}}

    st0 = stats[0]
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8 (decode) / bf16 x bf16 -> fp32 (gemm)",
        "data": "synthetic",
        "config": {"workload": args.workload, "N": N, "K": K, "Ms": list(Ms),
                   "pipelines": list(PIPES), "weight_sets": N_SETS,
                   "l2": f"{N_SETS} weight sets rotated per pipeline run, inputs > L2",
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "bits_per_exponent": st0["bits_per_exponent"],
                   "escape_row_fraction": st0["n_escape_rows"] / st0["n_rows"]},
        "roofline": roofline,
        "kernels": kernels,
        "pipelines": pipelines,
        "torch_matmul_bf16_us": tm,
        "back_to_back_us": b2b,
        "gemm_large_m": gemm_large,
        "huffman_direct": hdot,
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
        "kernel_src_sha": _kernel_src_sha(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    for h in handles:
        h.free()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_only(args):
    """Three launches of one kernel on the bench workload (first set of weights),
    for a profiler to capture (select by kernel name: decode_kernel<0|1|2> is
    exponent / full / transcode, decode_kernel<3> the Huffman-direct product,
    gemm_kernel<0|1|2> bf16 / exponent / palette, gemv_kernel<0|1|2, tokens>
    the matrix-vector kernels).
    The handle is uploaded without the load-time transcode unless the palette
    GEMM needs it (that launch comes first)."""
    import numpy as np
    import torch
    import decode_gemm_b200 as uw
    import synthdata

    w = synthdata.workload(args.workload)
    N, K = w.shape
    direct = args.only in ("gemm_palette", "gemv_palette")
    h = uw.uw_encode(w, uw.default_opts(prepare_direct=1 if direct else 0))
    out = torch.empty(2 * N * K, dtype=torch.uint8, device="cuda")
    pipe = {"gemm_bf16": 1, "gemm_exp": 2, "gemm_palette": 4,
            "gemv_bf16": 1, "gemv_exp": 2, "gemv_palette": 4, "decode_dot": 5}.get(args.only)
    gemv = args.only.startswith("gemv")
    if pipe:
        M = args.m
        X = torch.from_numpy(synthdata.activations(M, K, seed=11 + M).view(np.int16)).cuda()
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(uw.uw_workspace_bytes(h, pipe, M), dtype=torch.uint8, device="cuda")
        uw.uw_set_workspace(h, ws)
    for _ in range(3):
        if args.only == "decode_full":
            uw.uw_decode_full(h, out)
        elif args.only == "decode_exp":
            uw.uw_decode_exp(h, out)
        elif args.only == "transcode":
            uw.uw_transcode_palette(h, out)
        elif gemv:  # the CUDA-core matrix-vector kernel (M <= 2)
            uw.uw_gemm_ex(h, X, Y, M, uw.gemm_config(pipe, gemv=1), False)
        else:  # pipelines 1 and 2 run their decode first (select the GEMM by name)
            uw.uw_gemm(h, X, Y, M, pipe)
    torch.cuda.synchronize()
    if uw.uw_last_device_status(h) != uw.UW_OK:
        raise SystemExit("device status not OK")
    print(json.dumps({"only": args.only, "m": args.m if pipe else None, "launches": 3}))
    return 0


def run_mlp(args):
    """The 32-layer (or --mlp-layers) MLP stack: gate/up 14336x4096 and down
    4096x14336 per layer, BF16 ~ N(0, 0.02) with independent seeds, SiLU(gate)
    * up -> down.  Layer 0's projections are autotuned per M and the profile is
    applied to every layer; uw_mlp_tune_split picks the preprocessing overlap
    and SM split; uw_mlp_forward is timed with CUDA events (inputs resident)
    against the same stack in torch on the uncompressed BF16 weights."""
    import tempfile
    import numpy as np
    import torch
    import decode_gemm_b200 as uw
    import synthdata

    L = args.mlp_layers
    Ms = [int(m) for m in args.mlp_ms.split(",")]
    D, F = 4096, 14336
    torch.cuda.set_device(0)
    layers, wbf = [], []
    comp = bf = 0
    for i in range(L):
        trio, bfs = [], []
        for j, (n, k) in enumerate(((F, D), (F, D), (D, F))):
            w = synthdata.normal(n, k, 0.02, 2000 + 3 * i + j)
            h = uw.uw_encode(w)
            st = h.stats()
            comp += st["bytes_palette_bundle"] + st["bytes_stream"] + st["bytes_offsets"]
            bf += 2 * n * k
            trio.append(h)
            bfs.append(torch.from_numpy(w.view(np.int16)).cuda().view(torch.bfloat16))
            del w
        layers.append(tuple(trio))
        wbf.append(bfs)
    side = torch.cuda.Stream()
    if args.mlp_force_down:
        return _mlp_overlap_modes(args, uw, torch, np, synthdata, layers, wbf, Ms, D, side, bf,
                                  comp)
    flat0 = list(layers[0])
    need = max(uw.uw_workspace_bytes(h, p, max(Ms)) for h in flat0 for p in (1, 2, 3, 4))
    ws0 = torch.empty(need, dtype=torch.uint8, device="cuda")
    for h in flat0:
        uw.uw_set_workspace(h, ws0)
    with tempfile.TemporaryDirectory() as d:
        prof = os.path.join(d, "profile.json")
        uw.uw_autotune(flat0, Ms, prof)
        for trio in layers[1:]:
            uw.uw_load_profile(list(trio), prof)
    out = {}
    for M in Ms:
        x = synthdata.activations(M, D, 3000 + M)
        X = torch.from_numpy(x.view(np.int16)).cuda()
        Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
        ws = torch.empty(max(uw.uw_mlp_workspace_bytes(layers, M, uw.mlp_opts(o))
                             for o in (False, True)), dtype=torch.uint8, device="cuda")
        best = uw.uw_mlp_tune_split(layers, X, Y, M, ws, side_stream=side)

        def timed(fn, it=5):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(it):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / it

        ours = timed(lambda: uw.uw_mlp_forward(layers, X, Y, M, ws, best, side_stream=side))
        xb = X.view(torch.bfloat16)

        def ref():
            cur = xb
            for g, u, dw in wbf:
                a, b = cur @ g.t(), cur @ u.t()
                cur = (torch.nn.functional.silu(a.float()) * b.float()).to(torch.bfloat16) @ dw.t()
            return cur

        base = timed(ref)
        for h in flat0:
            if uw.uw_last_device_status(h) != uw.UW_OK:
                raise RuntimeError("device status")
        out[f"M{M}"] = {"ms": ours, "torch_bf16_ms": base, "ratio": ours / base,
                        "pipelines": [uw.uw_get_choice(h, M)["pipeline"] for h in flat0],
                        "split": best.as_dict()}
    print(json.dumps({"mode": "mlp_stack", "layers": L, "unit": "ms per forward",
                      "weights_bf16_bytes": bf, "weights_compressed_bytes": comp,
                      "data": "synthetic", "results": out}), flush=True)
    for trio in layers:
        for h in trio:
            h.free()
    return 0


def _mlp_overlap_modes(args, uw, torch, np, synthdata, layers, wbf, Ms, D, side, bf, comp):
    """The stack with every down_proj forced onto a hard pipeline (one that
    needs Huffman preprocessing) and gate/up on pipeline 4 (*Unweight*,
    "Sharing the GPU between decode and compute": down_proj gains most from
    overlapping its preprocessing).  For each M: the forward with the
    preprocessing serial on the main stream, overlapped on a side stream (all
    SMs for each kernel), and with the SM split uw_mlp_tune_split picks;
    torch BF16 on the uncompressed weights for context."""
    import json as _json
    import tempfile
    results = {}
    for pd in [int(x) for x in args.mlp_force_down.split(",") if x]:
        per_m = {}
        for M in Ms:
            prof = {"version": 1, "handles": []}
            for trio in layers:
                for h, p in zip(trio, (4, 4, pd)):
                    prof["handles"].append({"N": h.N, "K": h.K, "choices": [
                        {"M": M, "pipeline": p, "tile_n": 0, "stages": 0, "gemm_ctas": 0,
                         "decode_ctas": 0}]})
            with tempfile.NamedTemporaryFile("w", suffix=".json", delete=False) as f:
                _json.dump(prof, f)
                path = f.name
            uw.uw_load_profile([h for trio in layers for h in trio], path)
            os.unlink(path)
            x = synthdata.activations(M, D, 3000 + M)
            X = torch.from_numpy(x.view(np.int16)).cuda()
            Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
            ws = torch.empty(max(uw.uw_mlp_workspace_bytes(layers, M, uw.mlp_opts(o))
                                 for o in (False, True)), dtype=torch.uint8, device="cuda")

            def timed(fn, it=5):
                for _ in range(2):
                    fn()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(it):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                return e0.elapsed_time(e1) / it

            serial = timed(lambda: uw.uw_mlp_forward(layers, X, Y, M, ws, uw.mlp_opts(False),
                                                     side_stream=side))
            overlap = timed(lambda: uw.uw_mlp_forward(layers, X, Y, M, ws, uw.mlp_opts(True),
                                                      side_stream=side))
            best = uw.uw_mlp_tune_split(layers, X, Y, M, ws, side_stream=side)
            tuned = timed(lambda: uw.uw_mlp_forward(layers, X, Y, M, ws, best, side_stream=side))
            xb = X.view(torch.bfloat16)

            def ref():
                cur = xb
                for g, u, dw in wbf:
                    a, b = cur @ g.t(), cur @ u.t()
                    cur = (torch.nn.functional.silu(a.float()) * b.float()).to(torch.bfloat16) \
                        @ dw.t()
                return cur

            base = timed(ref)
            for trio in layers:
                for h in trio:
                    if uw.uw_last_device_status(h) != uw.UW_OK:
                        raise RuntimeError("device status")
            per_m[f"M{M}"] = {"serial_ms": serial, "overlap_ms": overlap, "tuned_split_ms": tuned,
                              "tuned_split": best.as_dict(), "torch_bf16_ms": base,
                              "overlap_gain": serial / overlap, "tuned_gain": serial / tuned}
        results[f"down_pipeline_{pd}"] = per_m
    print(json.dumps({"mode": "mlp_overlap", "layers": len(layers), "unit": "ms per forward",
                      "gate_up_pipeline": 4, "weights_bf16_bytes": bf,
                      "weights_compressed_bytes": comp, "data": "synthetic",
                      "results": results}), flush=True)
    for trio in layers:
        for h in trio:
            h.free()
    return 0


def main():
    args = _args()
    if args.only:
        return run_only(args)
    if args.mlp_layers > 0:
        return run_mlp(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
