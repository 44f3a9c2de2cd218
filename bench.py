#!/usr/bin/env python
"""Benchmark of the TQ3 KV-cache codec (and, on request, the RPBH weight path) on B200.

Default workload: a bf16 KV cache, K and V each [batch 8, kv_heads 8, seq 4096, head_dim 128]
(524,288 vectors of 128), N(0,1) plus 4 outlier channels x20 and a per-token N(0, 2^2) offset,
seed 1. One step encodes K and V to TQ3 records and decodes both back to bf16:
encode(K), encode(V), decode(K), decode(V). Inputs are resident in HBM; every kernel reads data
last touched at least one 160 MB kernel earlier, so no input is served from the 126 MB L2.

Prints ONE JSON line (rank 0). `value` = vectors encoded and decoded per second over all ranks
(each rank runs its own full cache: weak scaling, no data-path collective). `e2e` is the same
metric with K and V copied in from pinned host memory and the decoded caches plus the TQ3 records
copied back every step. `cpu_baseline` times the single-threaded C oracle on a bounded sample of
the same workload on this host. `--impl reference` times that oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_quantization_b200 import inputs  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
HBM_FALLBACK_GBS = 6650.0


# ---------------------------------------------------------------------------------------------
# environment helpers
# ---------------------------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return HBM_FALLBACK_GBS, "fallback"


def host_cpu():
    """The host's CPU model and the number of cores this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        nproc = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        nproc = os.cpu_count()
    return {"cpu": model or "unknown", "nproc": nproc}


class OneCore:
    """Runs the single-threaded oracle pinned to one of this process's cores, when the host allows
    it (`pinned` says whether it did); the affinity is restored afterwards."""

    def __enter__(self):
        self.saved, self.pinned = None, False
        try:
            self.saved = os.sched_getaffinity(0)
            os.sched_setaffinity(0, {min(self.saved)})
            self.pinned = True
        except (AttributeError, OSError, ValueError):
            pass
        return self

    def __exit__(self, *exc):
        if self.pinned:
            os.sched_setaffinity(0, self.saved)
        return False


def measured_tensor_peak():
    """Dense bf16 TFLOP/s measured on this machine (a cuBLAS burst), or the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.lines:
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def traffic_bytes(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` in `workload` from the committed ncu summary, if one was
    taken on that workload and on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    src = {"tq3_encode": "tq3_mma.cu", "tq3_decode": "tq3_rows.cu", "tq3_encode_exact": "tq3.cu",
           "rpbh_quantize": "rpbh_lanes.cu", "rpbh_rotate": "rpbh_lanes.cu", "rpbh_dequantize": "rpbh_fast.cu",
           "rpbh_linear": "rpbh_linear.cu", "tq3_attention": "tq3_attn.cu"}.get(kernel)
    if src is None:
        return None
    with open(os.path.join(ROOT, "weight_quantization_b200", "csrc", src), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    with open(p) as f:
        for line in f:
            parts = line.split()
            if (len(parts) >= 5 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload
                    and parts[2] == sha):
                return float(parts[4])
    return None


class Pipeline:
    """End-to-end steps over n units in `chunks` pieces on three streams (copy in, kernels, copy
    out). Piece i is copied in, processed and copied out in that order, while the copy in of piece
    i + 1 and the copy out of piece i - 1 overlap piece i's kernels (host-device copies run both
    directions at once). Consecutive steps overlap too: a piece's device buffers are reused as soon
    as that piece of the previous step is done with them (its copy in waits for the previous step's
    kernels on the piece, its kernels for the previous step's copy out), so the first pieces of a
    step run under the last pieces of the one before. Every step waits for the work the caller
    enqueued before it; `join` makes the caller's stream wait for all steps."""

    def __init__(self, dev, chunks):
        self.streams = [torch.cuda.Stream(dev) for _ in range(3)]
        self.chunks = chunks
        self.read = [None] * chunks     # piece i: the last step's kernels have read its inputs
        self.written = [None] * chunks  # piece i: the last step's copies out have read its outputs

    def step(self, n, h2d, compute, d2h):
        s_in, s_c, s_out = self.streams
        cur = torch.cuda.current_stream()
        for s in self.streams:
            s.wait_stream(cur)
        for i in range(self.chunks):
            a, b = i * n // self.chunks, (i + 1) * n // self.chunks
            with torch.cuda.stream(s_in):
                if self.read[i] is not None:
                    s_in.wait_event(self.read[i])
                h2d(a, b)
            s_c.wait_stream(s_in)
            with torch.cuda.stream(s_c):
                if self.written[i] is not None:
                    s_c.wait_event(self.written[i])
                compute(a, b)
                self.read[i] = torch.cuda.Event()
                self.read[i].record(s_c)
            s_out.wait_stream(s_c)
            with torch.cuda.stream(s_out):
                d2h(a, b)
                self.written[i] = torch.cuda.Event()
                self.written[i].record(s_out)

    def join(self):
        cur = torch.cuda.current_stream()
        for s in self.streams:
            cur.wait_stream(s)


E2E_CHUNKS = 8

# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------
class KVWorkload:
    """TQ3 encode + decode of a bf16 KV cache: K and V stored as one contiguous [2, 8, 8, 4096, 128]
    tensor, so one encode and one decode call cover all 524,288 vectors."""

    name = "tq3-kv-cache-bf16-2x8x8x4096x128"
    unit = "vectors/s"
    metric = "TQ3 encode+decode vectors/s (K and V caches, bf16)"

    def __init__(self, dev, seed=1):
        from weight_quantization_b200 import ops
        self.ops = ops
        k, v = inputs.kv_cache(seed=seed)
        kv = np.concatenate([k.reshape(-1, 128), v.reshape(-1, 128)])
        self.host = [torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16)]
        self.n_half = self.host[0].shape[0] // 2
        self.units = 2 * self.n_half
        n = self.units
        self.mask = ops.sign_mask_words(inputs.tq3_sign_bits())
        self.x = [self.host[0].to(dev)]
        # The records (29 MB, smaller than L2) rotate over RSETS sets: launch or step k encodes into
        # set k and decodes set k + 1, written RSETS - 1 launches earlier, so no decode reads
        # records that are still in L2 (the 134 MB cache itself is larger than L2).
        R = self.RSETS
        self.packed = [torch.empty(n, 48, dtype=torch.uint8, device=dev) for _ in range(R)]
        self.norms = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(R)]
        self.scales = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(R)]
        self.out = [torch.empty(n, 128, dtype=torch.bfloat16, device=dev)]
        for k in range(R):
            self._encode(k)
        # 56-byte records (timed beside the step), rotating over R sets as well; the paged forms
        # use pages of 16 records in a random page order
        self.recs = [ops.tq3_encode_aos(self.x[0], self.mask).view(n, 56) for _ in range(R)]
        self.page = 16
        g = torch.Generator().manual_seed(seed)
        self.table = torch.randperm(n // self.page, generator=g).to(torch.int32).to(dev)
        pos = torch.arange(n, dtype=torch.int64)
        self.slots = (self.table.cpu().to(torch.int64)[pos // self.page] * self.page + pos % self.page).to(dev)
        # the same cache as fp32 (268 MB, larger than L2), for the fp32-input encoder beside the step
        self.x32 = self.x[0].float()
        self.kernels = ["tq3_encode", "tq3_decode"]
        self.bytes_per_launch = {"tq3_encode": 312 * n, "tq3_decode": 312 * n, "tq3_encode_aos": 312 * n,
                                 "tq3_decode_aos": 312 * n, "tq3_encode_slots": 320 * n,
                                 "tq3_decode_paged": (312 + 4 / self.page) * n, "tq3_encode_fp32": 568 * n}
        self.l2 = (f"cache (134 MB) larger than L2; records rotate over {R} sets: launch k encodes into "
                   f"set k % {R} and decodes set (k + 1) % {R}, written {R - 1} launches earlier")

    RSETS = 8
    rotation = RSETS  # the buffer choice repeats every `rotation` steps

    def _encode(self, k, exact=False):
        r = k % self.RSETS
        self.ops.tq3_encode(self.x[0], self.mask, self.packed[r].view(-1, 1, 48), self.norms[r].view(-1, 1),
                            self.scales[r].view(-1, 1), exact=exact)

    def _decode(self, k):
        r = (k + 1) % self.RSETS
        self.ops.tq3_decode(self.packed[r], self.norms[r], self.scales[r], self.mask, out=self.out[0])

    def parts(self):
        """(kernel, launches, fn(k)) in step order: encode the cache, then decode it; k is the step
        (or launch) index, which picks the rotating buffers."""
        return [("tq3_encode", 1, self._encode), ("tq3_decode", 1, self._decode)]

    def extras(self):
        """Kernels timed beside the step (not part of it): the bit-exact encoder on the same cache, the
        encoder on the cache as fp32 input, and the codec on 56-byte records."""
        o, R = self.ops, self.RSETS
        return [("tq3_encode_exact", 1, lambda k: self._encode(k, exact=True)),
                ("tq3_encode_fp32", 1, lambda k: o.tq3_encode(self.x32, self.mask, self.packed[k % R].view(-1, 1, 48),
                                                               self.norms[k % R].view(-1, 1),
                                                               self.scales[k % R].view(-1, 1))),
                ("tq3_encode_aos", 1, lambda k: o.tq3_encode_aos(self.x[0], self.mask, records=self.recs[k % R])),
                ("tq3_decode_aos", 1, lambda k: o.tq3_decode_aos(self.recs[(k + 1) % R], self.mask,
                                                                 out_dtype=torch.bfloat16, out=self.out[0])),
                ("tq3_encode_slots", 1, lambda k: o.tq3_encode_slots(self.x[0], self.mask, self.slots,
                                                                     self.recs[k % R])),
                ("tq3_decode_paged", 1, lambda k: o.tq3_decode_paged(self.recs[(k + 1) % R], self.table, self.page,
                                                                     self.units, self.mask, out_dtype=torch.bfloat16,
                                                                     out=self.out[0]))]

    def step(self, k=0):
        for _, _, fn in self.parts():
            fn(k)

    # end to end: pinned host cache in; decoded cache and the TQ3 records out
    def e2e_setup(self):
        self.pin_in = [h.pin_memory() for h in self.host]
        self.pin_out = [torch.empty_like(h).pin_memory() for h in self.host]
        self.pin_packed = [torch.empty(self.units, 48, dtype=torch.uint8).pin_memory()]
        self.pin_ns = [torch.empty(2, self.units, dtype=torch.float32).pin_memory()]
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.pin_out + self.pin_packed + self.pin_ns)

        self.pipe = Pipeline(self.x[0].device, E2E_CHUNKS)

    def e2e_step(self):
        """The cache in from pinned memory, encoded and decoded through the public calls, the
        decoded cache and the records out, in E2E_CHUNKS pieces pipelined over three streams."""
        o = self.ops

        def h2d(a, b):
            self.x[0][a:b].copy_(self.pin_in[0][a:b], non_blocking=True)

        def compute(a, b):
            o.tq3_encode(self.x[0][a:b], self.mask, self.packed[0][a:b].view(-1, 1, 48),
                         self.norms[0][a:b].view(-1, 1), self.scales[0][a:b].view(-1, 1))
            o.tq3_decode(self.packed[0][a:b], self.norms[0][a:b], self.scales[0][a:b], self.mask,
                         out=self.out[0][a:b])

        def d2h(a, b):
            self.pin_out[0][a:b].copy_(self.out[0][a:b], non_blocking=True)
            self.pin_packed[0][a:b].copy_(self.packed[0][a:b], non_blocking=True)
            self.pin_ns[0][0][a:b].copy_(self.norms[0][a:b], non_blocking=True)
            self.pin_ns[0][1][a:b].copy_(self.scales[0][a:b], non_blocking=True)

        self.pipe.step(self.units, h2d, compute, d2h)

    def e2e_join(self):
        self.pipe.join()

    def e2e_check(self):
        """After the timed region: the host copies equal the device results."""
        return (torch.equal(self.pin_out[0], self.out[0].cpu()) and torch.equal(self.pin_packed[0], self.packed[0].cpu())
                and torch.equal(self.pin_ns[0][0], self.norms[0].cpu()) and torch.equal(self.pin_ns[0][1], self.scales[0].cpu()))

    # the oracle on a bounded sample of the same cache
    def oracle_rate(self, budget_s=10.0):
        import oracle
        oracle.lib()
        bits = inputs.tq3_sign_bits()
        src = self.host[0].view(torch.int16).numpy().view(np.uint16)
        done, t0, chunk = 0, time.perf_counter(), 2048
        while time.perf_counter() - t0 < budget_s:
            lo = done % (src.shape[0] - chunk)
            x = src[lo:lo + chunk]
            p, n, s = oracle.tq3_encode(x, bits, is_bf16=True)
            oracle.tq3_decode(p, n, s, bits, out_bf16=True)
            done += chunk
        dt = time.perf_counter() - t0
        return done / dt, f"{done} vectors of the K cache (cycling from the start), encode + decode to bf16, {dt:.1f} s"


class LongContextWorkload(KVWorkload):
    """Decode-only: 1,048,576 TQ3 records to bf16 [1, 8, 131072, 128]."""

    name = "tq3-decode-long-context-1x8x131072x128"
    metric = "TQ3 decode vectors/s (1M records to bf16)"

    def __init__(self, dev, seed=2):
        from weight_quantization_b200 import ops
        self.ops = ops
        p, n, s = inputs.long_context_records(seed=seed)
        self.mask = ops.sign_mask_words(inputs.tq3_sign_bits())
        self.host_rec = (torch.from_numpy(p), torch.from_numpy(n), torch.from_numpy(s))
        # the records (59 MB, smaller than L2) rotate over RSETS copies, one per launch
        self.recs = [[t.to(dev) for t in self.host_rec] for _ in range(self.RSETS)]
        self.rec = self.recs[0]
        self.n_half = p.shape[0]
        self.units = self.n_half
        self.out = torch.empty(self.n_half, 128, dtype=torch.bfloat16, device=dev)
        self.kernels = ["tq3_decode"]
        self.bytes_per_launch = {"tq3_decode": 312 * self.n_half}
        self.l2 = (f"records rotate over {self.RSETS} copies ({self.RSETS} x 59 MB, larger than L2), launch k "
                   f"decoding copy k % {self.RSETS}")

    RSETS = 4
    rotation = RSETS

    def parts(self):
        def dec(k):
            r = self.recs[k % self.RSETS]
            self.ops.tq3_decode(r[0], r[1], r[2], self.mask, out=self.out)
        return [("tq3_decode", 1, dec)]

    def extras(self):
        return []

    def e2e_setup(self):
        self.pin_rec = [t.pin_memory() for t in self.host_rec]
        self.pin_out = torch.empty(self.n_half, 128, dtype=torch.bfloat16).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin_rec)
        self.d2h = self.pin_out.numel() * 2
        self.pipe = Pipeline(self.out.device, E2E_CHUNKS)

    step = KVWorkload.step
    e2e_join = KVWorkload.e2e_join

    def e2e_step(self):
        """The records in from pinned memory, decoded through the public call, the bf16 cache out,
        in E2E_CHUNKS pieces pipelined over three streams."""
        def h2d(a, b):
            for d, h in zip(self.rec, self.pin_rec):
                d[a:b].copy_(h[a:b], non_blocking=True)

        def compute(a, b):
            self.ops.tq3_decode(self.rec[0][a:b], self.rec[1][a:b], self.rec[2][a:b], self.mask, out=self.out[a:b])

        def d2h(a, b):
            self.pin_out[a:b].copy_(self.out[a:b], non_blocking=True)

        self.pipe.step(self.units, h2d, compute, d2h)

    def e2e_check(self):
        return torch.equal(self.pin_out, self.out.cpu())

    def oracle_rate(self, budget_s=10.0):
        import oracle
        oracle.lib()
        bits = inputs.tq3_sign_bits()
        p, n, s = (t.numpy() for t in self.host_rec)
        done, t0, chunk = 0, time.perf_counter(), 4096
        while time.perf_counter() - t0 < budget_s and done + chunk <= p.shape[0]:
            oracle.tq3_decode(p[done:done + chunk], n[done:done + chunk], s[done:done + chunk], bits, out_bf16=True)
            done += chunk
        dt = time.perf_counter() - t0
        return done / dt, f"first {done} records decoded to bf16, {dt:.1f} s"


class RPBHWorkload:
    """RPBH on an LLM MLP weight W[4096, 11008] bf16 (3 bits) and activations x[2048, 11008]:
    quantize W, dequantize W' (rotated, bf16) and rotate x."""

    metric = "RPBH weight elements/s (quantize + rotated dequantize + activation rotation)"
    unit = "elements/s"

    def __init__(self, dev, rows=4096, d=11008, xrows=2048, bits=3, seed=3, name=None):
        from weight_quantization_b200 import ops
        self.ops = ops
        self.name = name or f"rpbh-w{rows}x{d}-x{xrows}-b{bits}"
        w = inputs.llm_weight(rows, d, seed=seed) if d == 11008 else inputs.dit_weight(rows, d, seed=seed)
        x = inputs.activations(xrows, d, seed=seed)
        perm, signs = inputs.rpbh_params(d)
        self.rows, self.d, self.xrows, self.bits = rows, d, xrows, bits
        bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        self.host = [bf(w), bf(x)]
        # W (75-90 MB), x (25-45 MB) and the codes (14-17 MB) are smaller than L2: each rotates over
        # copies, so a launch reads data last touched several hundred MB of traffic earlier
        W, X, P = self.WSETS, self.XSETS, self.PSETS
        self.ws = [self.host[0].to(dev) for _ in range(W)]
        self.xs = [self.host[1].to(dev) for _ in range(X)]
        self.w, self.x = self.ws[0], self.xs[0]
        self.perm = torch.from_numpy(perm).to(dev)
        self.signs = torch.from_numpy(signs).to(dev)
        self.cb = ops.rpbh_codebook(bits, d)
        self.packeds = [torch.empty(ops.rpbh_packed_bytes(rows, d, bits), dtype=torch.uint8, device=dev)
                        for _ in range(P)]
        self.normss = [torch.empty(rows, dtype=torch.bfloat16, device=dev) for _ in range(P)]
        self.packed, self.norms = self.packeds[0], self.normss[0]
        self.wq = torch.empty(rows, d, dtype=torch.bfloat16, device=dev)
        self.xr = torch.empty(xrows, d, dtype=torch.bfloat16, device=dev)
        for k in range(P):
            self._quantize(k)
        self.units = rows * d
        self.kernels = ["rpbh_quantize", "rpbh_dequantize", "rpbh_rotate"]
        n = rows * d
        self.bytes_per_launch = {"rpbh_quantize": 2 * n + n * bits // 8 + 2 * rows,
                                 "rpbh_dequantize": 2 * n + n * bits // 8 + 2 * rows,
                                 "rpbh_rotate": 4 * xrows * d}
        self.l2 = (f"W rotates over {W} copies, x over {X}, the codes over {P} sets: launch k quantizes W "
                   f"copy k % {W} into set k % {P}, dequantizes set (k + 1) % {P} (written {P - 1} launches "
                   f"earlier) and rotates x copy k % {X}")

    WSETS, XSETS, PSETS = 3, 4, 3
    rotation = 12  # lcm of the three

    def _quantize(self, k):
        p = k % self.PSETS
        self.ops.rpbh_quantize_weight(self.ws[k % self.WSETS], self.perm, self.signs, self.bits, self.cb,
                                      self.packeds[p], self.normss[p])

    def parts(self):
        o = self.ops

        def rot(k):
            o.rpbh_rotate_activations(self.xs[k % self.XSETS], self.perm, self.signs, out=self.xr)

        def deq(k):
            p = (k + 1) % self.PSETS
            o.rpbh_dequantize_weight(self.packeds[p], self.normss[p], self.rows, self.d, self.bits, self.cb,
                                     out_dtype=torch.bfloat16, out=self.wq)

        return [("rpbh_quantize", 1, self._quantize), ("rpbh_rotate", 1, rot), ("rpbh_dequantize", 1, deq)]

    step = KVWorkload.step

    def e2e_setup(self):
        self.pin_in = [h.pin_memory() for h in self.host]
        self.pin_out = [torch.empty_like(self.wq, device="cpu").pin_memory(),
                        torch.empty_like(self.xr, device="cpu").pin_memory()]
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.pin_out)

    def e2e_step(self):
        o = self.ops
        self.w.copy_(self.pin_in[0], non_blocking=True)
        self.x.copy_(self.pin_in[1], non_blocking=True)
        o.rpbh_quantize_weight(self.w, self.perm, self.signs, self.bits, self.cb, self.packed, self.norms)
        o.rpbh_rotate_activations(self.x, self.perm, self.signs, out=self.xr)
        o.rpbh_dequantize_weight(self.packed, self.norms, self.rows, self.d, self.bits, self.cb,
                                 out_dtype=torch.bfloat16, out=self.wq)
        self.pin_out[0].copy_(self.wq, non_blocking=True)
        self.pin_out[1].copy_(self.xr, non_blocking=True)

    def oracle_rate(self, budget_s=10.0):
        import oracle
        oracle.lib()
        perm, signs = inputs.rpbh_params(self.d)
        h = self.d & -self.d
        w = self.host[0].view(torch.int16).numpy().view(np.uint16)
        cb = self.cb
        done, t0, chunk = 0, time.perf_counter(), 32
        while time.perf_counter() - t0 < budget_s and done + chunk <= self.rows:
            p, n = oracle.rpbh_quantize(w[done:done + chunk], perm, signs, h, cb, self.bits, is_bf16=True)
            oracle.rpbh_dequantize_rotated(p, n, chunk, self.d, self.bits, cb, out_bf16=True)
            done += chunk
        dt = time.perf_counter() - t0
        return done * self.d / dt, f"first {done} weight rows quantized + dequantized (no activations), {dt:.1f} s"


class RPBHLinearWorkload:
    """The fused RPBH linear layer of forward on the LLM MLP shape: y[2048, 4096] = x_rot W'^T + b,
    W'[4096, 11008] held as 3-bit codes and row norms (from quantizing the LLM weight), x_rot bf16."""

    metric = "RPBH fused dequantize + linear FLOP/s (2 m n d per call)"
    unit = "FLOP/s"
    bound = "tensor"

    def __init__(self, dev, out_f=4096, d=11008, m=2048, bits=3, seed=5):
        from weight_quantization_b200 import ops
        self.ops = ops
        self.name = f"rpbh-linear-w{out_f}x{d}-x{m}-b{bits}"
        self.out_f, self.d, self.m, self.bits = out_f, d, m, bits
        bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        perm, signs = inputs.rpbh_params(d)
        perm_d, signs_d = torch.from_numpy(perm).to(dev), torch.from_numpy(signs).to(dev)
        w = bf(inputs.llm_weight(out_f, d, seed=seed)).to(dev)
        self.cb = ops.rpbh_codebook(bits, d)
        packed, norms = ops.rpbh_quantize_weight(w, perm_d, signs_d, bits, self.cb)
        del w
        x = bf(inputs.activations(m, d, seed=seed)).to(dev)
        xr = ops.rpbh_rotate_activations(x, perm_d, signs_d)
        # x_rot (45 MB) and the codes (17 MB) are smaller than L2: each rotates over copies
        X, P = self.XSETS, self.PSETS
        self.xs = [xr.clone() for _ in range(X)]
        self.packeds = [packed.clone() for _ in range(P)]
        self.norms = norms
        self.bias = (torch.randn(out_f, generator=torch.Generator().manual_seed(seed)) * 0.01).to(torch.bfloat16).to(dev)
        self.y = torch.empty(m, out_f, dtype=torch.bfloat16, device=dev)
        self.host_x = xr.cpu()
        self.units = 2 * m * out_f * d
        self.kernels = ["rpbh_linear"]
        self.flops_per_launch = {"rpbh_linear": 2 * m * out_f * d}
        self.bytes_per_launch = {"rpbh_linear": packed.numel() + 2 * out_f + 2 * m * d + 2 * m * out_f + 2 * out_f}
        self.l2 = (f"x_rot rotates over {X} copies and the codes over {P} sets: launch k uses x_rot copy "
                   f"k % {X} and code set k % {P}")

    XSETS, PSETS = 4, 3
    rotation = 12

    def _linear(self, k, x=None):
        self.ops.rpbh_linear(self.packeds[k % self.PSETS], self.norms, self.out_f, self.d, self.bits, self.cb,
                             self.xs[k % self.XSETS] if x is None else x, bias=self.bias, out=self.y)

    def parts(self):
        return [("rpbh_linear", 1, self._linear)]

    def extras(self):
        return []

    step = KVWorkload.step

    def e2e_setup(self):
        self.pin_in = self.host_x.pin_memory()
        self.pin_out = torch.empty(self.m, self.out_f, dtype=torch.bfloat16).pin_memory()
        self.h2d = self.pin_in.numel() * 2
        self.d2h = self.pin_out.numel() * 2

    def e2e_step(self):
        """x_rot in from pinned memory, the layer through the public call, y out (the weight codes
        stay resident, as in serving)."""
        self.xs[0].copy_(self.pin_in, non_blocking=True)
        self._linear(0)
        self.pin_out.copy_(self.y, non_blocking=True)

    def oracle_rate(self, budget_s=10.0):
        import oracle
        oracle.lib()
        p = self.packeds[0].cpu().numpy()
        n32 = self.norms.float().cpu().numpy()
        x = self.host_x.view(torch.int16).numpy().view(np.uint16)
        b = self.bias.cpu().view(torch.int16).numpy().view(np.uint16)
        rows_w = 64  # output features per sample (whole rows of the packed stream)
        row_bytes = self.d // 8 * self.bits
        done, t0, flops = 0, time.perf_counter(), 0
        while time.perf_counter() - t0 < budget_s and (done + 1) * rows_w <= self.out_f:
            lo = done * rows_w
            oracle.rpbh_linear(p[lo * row_bytes:(lo + rows_w) * row_bytes], n32[lo:lo + rows_w], rows_w, self.d,
                               self.bits, self.cb, x[:64], b[lo:lo + rows_w])
            flops += 2 * 64 * rows_w * self.d
            done += 1
        dt = time.perf_counter() - t0
        return flops / dt, f"{done} blocks of 64 output features x 64 activation rows (dequantize + fp64 product), {dt:.1f} s"


class TQ3AttentionWorkload:
    """Decode-step attention over a TQ3 KV cache: 8 sequences x 8 KV heads x 32768 keys, 4 query rows
    per KV head (32 query heads, one token), bf16 queries and outputs. K and V are 56-byte records
    drawn with the long-context recipe (235 MB together, larger than L2)."""

    metric = "TQ3 attention keys/s (key-value records attended per second)"
    unit = "keys/s"

    def __init__(self, dev, heads=64, S=32768, m=4, seed=6):
        from weight_quantization_b200 import ops
        self.ops = ops
        self.name = f"tq3-attention-decode-{heads}x{S}-m{m}"
        self.heads, self.S, self.m = heads, S, m
        self.mask = ops.sign_mask_words(inputs.tq3_sign_bits())

        def records(sd):
            p, n, sc = (torch.from_numpy(a) for a in inputs.long_context_records(heads * S, seed=sd))
            return torch.cat([p, n.view(torch.uint8).view(-1, 4), sc.view(torch.uint8).view(-1, 4)], 1).view(heads, S, 56)

        self.kr, self.vr = records(seed).to(dev), records(seed + 1).to(dev)
        q = torch.randn(heads, m, 128, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
        self.host_q = q
        self.q = q.to(dev)
        self.out = torch.empty(heads, m, 128, dtype=torch.bfloat16, device=dev)
        self.units = heads * S
        self.kernels = ["tq3_attention"]
        self.bytes_per_launch = {"tq3_attention": 112 * heads * S + 2 * 2 * heads * m * 128}
        self.l2 = "K and V records (235 MB) larger than L2, read once per launch"

    rotation = 1

    def _attn(self, k):
        self.ops.tq3_attention(self.q, self.kr, self.vr, self.mask, out=self.out)

    def parts(self):
        return [("tq3_attention", 1, self._attn)]

    def extras(self):
        return []

    step = KVWorkload.step

    def e2e_setup(self):
        self.pin_in = self.host_q.pin_memory()
        self.pin_out = torch.empty(self.heads, self.m, 128, dtype=torch.bfloat16).pin_memory()
        self.h2d = self.pin_in.numel() * 2
        self.d2h = self.pin_out.numel() * 2

    def e2e_step(self):
        """The step's queries in from pinned memory, attention through the public call, the output
        rows out (the cache stays resident, as in decoding)."""
        self.q.copy_(self.pin_in, non_blocking=True)
        self._attn(0)
        self.pin_out.copy_(self.out, non_blocking=True)

    def e2e_check(self):
        return torch.equal(self.pin_out, self.out.cpu())

    def oracle_rate(self, budget_s=10.0):
        import oracle
        oracle.lib()
        bits = inputs.tq3_sign_bits()
        q = self.host_q.float().numpy()
        kr, vr = self.kr[:1].cpu().numpy(), self.vr[:1].cpu().numpy()
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < budget_s and done < 64:
            oracle.tq3_attention(q[:1], kr, vr, bits, 128 ** -0.5)
            done += 1
        dt = time.perf_counter() - t0
        return done * self.S / dt, f"{done} passes over head 0 ({self.S} keys, {self.m} query rows), {dt:.1f} s"


WORKLOADS = {
    "kv": KVWorkload,
    "tq3-attention": TQ3AttentionWorkload,
    "longctx": LongContextWorkload,
    "rpbh-llm": lambda dev: RPBHWorkload(dev),
    "rpbh-dit": lambda dev: RPBHWorkload(dev, rows=12288, d=3072, xrows=4096, bits=3, seed=4),
    "rpbh-linear": RPBHLinearWorkload,
}


# ---------------------------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over all ranks (the job's wall time is set by its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args):
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    if args.workload == "tq3-attention":
        wl = TQ3AttentionWorkload(dev, m=args.attn_rows)
    else:
        wl = WORKLOADS[args.workload](dev)
    parts = wl.parts()
    # eager warm-up (loads the library, sets kernel attributes). The timed steps are then replayed
    # from CUDA graphs that hold up to CHUNK consecutive steps each (host launch overhead and
    # per-graph launch gaps stay out of the timed region); events on the replay stream bracket the
    # whole region. Event-record nodes between kernels would add several microseconds to each
    # kernel, so per-kernel durations come from a second timed region below: one graph per kernel
    # of back-to-back launches on the same buffers, bracketed by events.
    wl.step(0)
    torch.cuda.synchronize()
    CHUNK = 500

    def capture(fns, n, k0=0):
        """A graph of n consecutive steps (or launches) k0 .. k0 + n - 1."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                for fn in fns:
                    fn(k0 + i)
        return g

    step_fns = [fn for _, _, fn in parts]
    warm = capture(step_fns, args.warmup)
    sizes = [CHUNK] * (args.steps // CHUNK) + ([args.steps % CHUNK] if args.steps % CHUNK else [])
    # the graphs continue the step index (which picks the rotating buffers) from one to the next
    chunks = [capture(step_fns, n, args.warmup + sum(sizes[:c])) for c, n in enumerate(sizes)]
    warm.replay()
    torch.cuda.synchronize()
    barrier(world)

    # timed region: exactly K steps
    launches = sum(n for _, n, _ in parts) * args.steps
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        e_start.record()
        for g in chunks:
            g.replay()
        e_end.record()
        torch.cuda.synchronize()
        barrier(world)
    ms_total = e_start.elapsed_time(e_end)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    value = world * wl.units * args.steps / (ms_total / 1e3)
    del warm, chunks

    # per-kernel durations (second timed region, same buffers): a whole number of buffer rotations,
    # so that the warm-up replay and the timed one continue the same periodic sequence
    per_kernel = {}
    rot = getattr(wl, "rotation", 1)
    reps = max(rot, (max(3, min(args.steps, 200)) // rot) * rot)
    for name, n, fn in parts:
        g = capture([fn], reps)
        g.replay()
        torch.cuda.synchronize()
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record()
        g.replay()
        k1.record()
        torch.cuda.synchronize()
        avg_ms = max_over_ranks(k0.elapsed_time(k1), world) / (n * reps)
        per_kernel[name] = {"avg_us": avg_ms * 1e3, "launches": n * reps,
                            "gbs": wl.bytes_per_launch[name] / (avg_ms / 1e3) / 1e9}
        del g
    dom = max(per_kernel, key=lambda k: per_kernel[k]["avg_us"] * per_kernel[k]["launches"])
    peak, peak_kind = measured_peaks()
    achieved = per_kernel[dom]["gbs"]

    # kernels reported beside the step (same inputs, timed the same way, not part of `value`)
    beside = {}
    for name, n, fn in (wl.extras() if hasattr(wl, "extras") else []):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(reps):
                fn(i)
        g.replay()  # warm-up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        avg_ms = e0.elapsed_time(e1) / (n * reps)
        beside[name] = {"avg_us": avg_ms * 1e3, "launches": n * reps,
                        "gbs": wl.bytes_per_launch.get(name, wl.bytes_per_launch[parts[0][0]]) / (avg_ms / 1e3) / 1e9}
        del g

    # end to end through the same API with pinned host buffers
    wl.e2e_setup()
    join = getattr(wl, "e2e_join", lambda: None)  # steps that overlap one another are joined once, before the end event
    for _ in range(max(1, args.warmup // 2)):
        wl.e2e_step()
    join()
    torch.cuda.synchronize()
    barrier(world)
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(2, min(args.steps, 10))
    es.record()
    for _ in range(e2e_steps):
        wl.e2e_step()
    join()
    ee.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(es.elapsed_time(ee), world)
    if hasattr(wl, "e2e_check") and not wl.e2e_check():
        raise RuntimeError("end-to-end step: the host copies differ from the device results")
    e2e_value = world * wl.units * e2e_steps / (e2e_ms / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with OneCore() as pin:
            rate, sample = wl.oracle_rate(args.cpu_seconds)
        cpu = {"value": rate, "unit": wl.unit, "cores": 1, "kind": "oracle", "sample": sample,
               "pinned": pin.pinned, **host_cpu()}

    if getattr(wl, "bound", "hbm") == "tensor":
        tpeak, tkind = measured_tensor_peak()
        tflops = wl.flops_per_launch[dom] / (per_kernel[dom]["avg_us"] * 1e-6) / 1e12
        roofline = {"bound": "tensor", "kernel": dom, "achieved": tflops, "peak": tpeak, "peak_kind": tkind,
                    "unit": "TFLOP/s", "frac": tflops / tpeak, "traffic": traffic_bytes(dom, args.workload),
                    "algorithmic_flops_per_launch": wl.flops_per_launch[dom],
                    "algorithmic_bytes_per_launch": wl.bytes_per_launch[dom]}
    else:
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                    "unit": "GB/s", "frac": achieved / peak, "traffic": traffic_bytes(dom, args.workload),
                    "algorithmic_bytes_per_launch": wl.bytes_per_launch[dom]}
    if rank == 0:
        line = {
            "metric": wl.metric, "value": value, "unit": wl.unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "units_per_step_per_gpu": wl.units,
                       "io_dtype": "bf16", "l2": wl.l2, "launch": f"CUDA graphs of up to 500 consecutive steps; per-kernel times from graphs of {reps} back-to-back launches",
                       "parallelism": f"replicas x{world} (no collective)"},
            "roofline": roofline,
            "kernels": per_kernel,
            **({"kernels_beside_step": beside} if beside else {}),
            "e2e": {"value": e2e_value, "unit": wl.unit, "h2d_bytes_per_step": wl.h2d,
                    "d2h_bytes_per_step": wl.d2h},
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The oracle, as it stands, on the host cores: the reference arm of this benchmark."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.lib()
    dev = torch.device("cpu")
    # build the workload's host data only (no device needed)
    if args.workload == "kv":
        k, _ = inputs.kv_cache()
        src = k.reshape(-1, 128)
        name, unit, metric = KVWorkload.name, KVWorkload.unit, KVWorkload.metric
        bits = inputs.tq3_sign_bits()
        chunk = args.ref_chunk

        def step(i):
            lo = (i * chunk) % (src.shape[0] - chunk)
            p, n, s = oracle.tq3_encode(src[lo:lo + chunk], bits, is_bf16=True)
            oracle.tq3_decode(p, n, s, bits, out_bf16=True)
            return chunk
    else:
        raise SystemExit(f"--impl reference supports the default workload only, not {args.workload}")
    with OneCore() as pin:
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        units = 0
        for i in range(args.steps):
            units += step(args.warmup + i)
        dt = time.perf_counter() - t0
    value = units / dt
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": name, "sample_vectors_per_step": chunk},
            "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle",
                             "sample": f"{chunk} vectors of the K cache per step, encode + decode",
                             "pinned": pin.pinned, **host_cpu()},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="kv")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-chunk", type=int, default=2048)
    ap.add_argument("--attn-rows", type=int, default=4,
                    help="query rows per KV head for --workload tq3-attention (1..16)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
