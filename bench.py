"""HQMQ KV-cache encode/decode throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl hqmq|reference]

One step = one pass of the per-batch hot path over the whole synthetic KV
cache of the workload, layer by layer: per (layer, role) call Med3x (median +
ordered outlier list, when the workload has it), encode, and decode back to
bf16.  The per-model setup (secondary codebooks of every (layer, role, head)
and their search tables) runs once before the timed region and is reported
as `setup_ms`.  Inputs are resident in HBM before the timed region (the
default workload's cache is 42.95 GB, far above L2).

Prints one JSON line.  `value` = bf16 KV bytes taken through encode and
decode per second, summed over ranks (every rank codes its own cache: weak
scaling, no collective on the data path).  `e2e` is the same metric through
the C ABI from pinned host buffers (input H2D and compressed cache D2H inside
the timed region).  `--impl reference` times the CPU oracle (the plain
reference implementation of the method) on a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "HQMQ encode/decode GB/s (bf16 KV) and % of B200 HBM roofline, S=8/32"
DEFAULT_WORKLOAD = "llama3_70b_128k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}
ALU_LANES = 148 * 128          # FP32 lanes of a B200 (148 SMs x 128)
# kernels per call: fused Med3x+encode = sample, window, full pass, final
# select, fallback check, uncertain fix-up, tile scan, list+encode pass
KERNELS_MED3_ENCODE = 4          # k_sample_window, k_pass_b, k_finalize, k_encode_lut
OUTLIER_CAP_FRAC = 0.15        # list capacity: 15% of the chunks of a call


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    import torch
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    import torch.distributed as dist
    import datetime
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                            device_id=torch.device("cuda", local))
    return dist.get_rank(), dist.get_world_size(), dist


def max_over_ranks(v, dist, device):
    """Max of a float over ranks (identity without a process group)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle-reason samples during the timed region, taken
    every 10 ms through NVML from a thread (nvidia-smi as a fallback), on the
    GPU that CUDA device `gpu_index` is (found by its PCI address: the CUDA
    index and the NVML index differ when CUDA_VISIBLE_DEVICES is set)."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        import torch
        self.gpu = str(gpu_index)
        self.proc = None
        self.thread = None
        self.nv = None
        self.path = "/tmp/hqmq_clocks_%d.csv" % os.getpid()
        try:
            pr = torch.cuda.get_device_properties(gpu_index)
            self.gpu = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        except Exception:
            pass
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(self.gpu)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(int(gpu_index))
            self.nv = pynvml
        except Exception:
            self.nv = None

    def _loop(self):
        nv, h = self.nv, self.h
        bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        while not self.halt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, [n for n, b in zip(self.NAMES, bits) if r & b]))
            except Exception:
                pass
            self.halt.wait(0.01)

    def start(self):
        if self.nv is not None:
            import threading
            self.samples = []
            self.halt = threading.Event()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.halt.set()
            self.thread.join(timeout=5)
            self.thread = None
            if not self.samples:
                return None
            try:
                mx = float(self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            except Exception:
                mx = 0.0
            reasons = sorted({n for _, rs in self.samples for n in rs})
            return {"sm_mhz": statistics.median(float(c) for c, _ in self.samples),
                    "sm_max_mhz": mx, "reasons": reasons, "samples": len(self.samples),
                    "source": "nvml, every 10 ms", "device": self.gpu}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(self.NAMES, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi", "device": self.gpu}


# ---------------------------------------------------------------- the path
class Cache:
    """Device-resident synthetic cache of one workload and its code buffers."""

    def __init__(self, w, rank, device):
        import torch
        from kv_cache_quantization_hqmq_b200 import hqmq
        from kv_cache_quantization_hqmq_b200 import workloads as W
        self.w = w
        B, H, T, D = w.call_shape
        self.shape = (B, H, T, D)
        self.n_chunks = B * H * T * D // 4
        self.n_words = hqmq.hqmq_index_words(B, H, T, D, w.S)
        # each rank codes its own cache (different input seed)
        wr = w.with_(input_seed=w.input_seed + 1000 * rank)
        self.x = torch.empty((w.layers, 2) + self.shape, dtype=w.torch_dtype, device=device)
        for l in range(w.layers):
            for r in range(2):
                self.x[l, r].copy_(W.make_call_input(wr, l, r, device=device))
        self.codebook = torch.empty(w.n_groups * w.S * 4, dtype=torch.float32, device=device)
        # exact table-driven search when S allows it (else the S-codeword loop)
        self.table_bytes = hqmq.hqmq_search_table_bytes(w.S)
        self.table = None
        if self.table_bytes:
            self.table = torch.empty(w.n_groups * self.table_bytes, dtype=torch.uint8,
                                     device=device)
        self.words = torch.empty((w.layers, 2, self.n_words), dtype=torch.int32, device=device)
        self.radius = torch.empty((w.layers, 2, self.n_chunks), dtype=torch.int16, device=device)
        self.y = torch.empty(self.shape, dtype=torch.bfloat16, device=device)
        self.status = hqmq.new_status(device)
        self.gran = hqmq.HQMQ_GRAN_CHUNK
        if w.med3:
            self.cap = int(OUTLIER_CAP_FRAC * self.n_chunks)
            self.rmed = torch.empty((w.layers, 2, H), dtype=torch.float32, device=device)
            self.thr = torch.empty((w.layers, 2, H), dtype=torch.float32, device=device)
            self.out_idx = torch.empty((w.layers, 2, self.cap), dtype=torch.int32, device=device)
            self.out_val = torch.empty((w.layers, 2, self.cap * 4), dtype=torch.int16, device=device)
            self.slab_off = torch.empty((w.layers, 2, B * H + 1), dtype=torch.int32, device=device)
            # list tile offsets (rows padded to 16 bytes: the library stores them as uint4)
            self.n_tiles = hqmq.hqmq_list_tiles(B, H, T, D)
            self.tile_off = torch.empty((w.layers, 2, (self.n_tiles + 4) // 4 * 4),
                                        dtype=torch.int32, device=device)
            self.ws = torch.empty(hqmq.hqmq_encode_med3_workspace_size(B, H, T, D, self.gran),
                                  dtype=torch.uint8, device=device)

    def setup(self):
        """Per-model work, outside the timed step: the secondary codebooks of
        every (layer, role, head) and their search tables.  Returns its device
        time in ms (CUDA events)."""
        import torch
        from kv_cache_quantization_hqmq_b200 import hqmq
        w = self.w
        stream = torch.cuda.current_stream()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        hqmq.hqmq_make_codebook(w.codebook_seed, w.S, w.n_groups, 0, self.codebook, stream)
        if self.table is not None:
            for g0 in range(0, w.n_groups, 65535):
                n = min(65535, w.n_groups - g0)
                hqmq.hqmq_make_search_table(self.codebook[g0 * w.S * 4:(g0 + n) * w.S * 4], w.S, n,
                                            self.table[g0 * self.table_bytes:
                                                       (g0 + n) * self.table_bytes], stream)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    def kernels_per_step(self):
        if self.w.med3:
            enc = KERNELS_MED3_ENCODE + (0 if self.table is not None else 1)
            dec = 1                        # the list is applied in the main pass (tile offsets)
        else:
            enc, dec = 1, 1
        return self.w.n_calls * (enc + dec)

    def step(self):
        """One pass over the cache: every (layer, role) call, on the current
        stream."""
        import torch
        w = self.w
        stream = torch.cuda.current_stream()
        for l in range(w.layers):
            for r in range(2):
                self.call(l, r, self.x[l, r], stream)

    def call(self, l, r, x, stream):
        """One (layer, role) call on `stream`: Med3x + encode, then decode."""
        self.encode_call(l, r, x, stream)
        self.decode_call(l, r, stream)

    def _groups(self, l, r):
        w = self.w
        g0 = (l * 2 + r) * w.heads
        cb = self.codebook[g0 * w.S * 4:(g0 + w.heads) * w.S * 4]
        tb = None
        if self.table is not None:
            tb = self.table[g0 * self.table_bytes:(g0 + w.heads) * self.table_bytes]
        return cb, tb

    def encode_call(self, l, r, x, stream):
        """Med3x + encode of one (layer, role) call."""
        from kv_cache_quantization_hqmq_b200 import hqmq
        w = self.w
        cb, tb = self._groups(l, r)
        if w.med3:
            # Med3x and encode in one fused call (one read of x in chunk mode
            # with search tables, two otherwise)
            hqmq.hqmq_encode_med3(x, w.C, self.gran, cb, w.S, tb, self.words[l, r],
                                  self.radius[l, r], self.rmed[l, r], self.thr[l, r],
                                  self.out_idx[l, r], self.out_val[l, r],
                                  self.slab_off[l, r], self.cap, self.ws, self.status,
                                  stream, tile_off=self.tile_off[l, r])
        elif self.table is not None:
            hqmq.hqmq_encode_lut(x, cb, w.S, tb, None, self.gran, self.words[l, r],
                                 self.radius[l, r], self.status, stream)
        else:
            hqmq.hqmq_encode(x, cb, w.S, None, self.gran, self.words[l, r],
                             self.radius[l, r], self.status, stream)

    def decode_call(self, l, r, stream):
        """Decode of one (layer, role) call into the reusable output buffer."""
        from kv_cache_quantization_hqmq_b200 import hqmq
        w = self.w
        cb, _ = self._groups(l, r)
        if w.med3:
            hqmq.hqmq_decode(self.words[l, r], self.radius[l, r], cb, w.S,
                             self.out_idx[l, r], self.out_val[l, r], self.slab_off[l, r],
                             self.cap, self.gran, self.y, self.status, stream,
                             tile_off=self.tile_off[l, r])
        else:
            hqmq.hqmq_decode(self.words[l, r], self.radius[l, r], cb, w.S, None, None,
                             None, 0, self.gran, self.y, self.status, stream)

    def capture(self, fn):
        """fn's launches captured in one CUDA graph (replayed once)."""
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        return g

    def graph_times(self, reps):
        """Device time of one step, of the step's encode calls and of its
        decode calls, each captured in one CUDA graph and replayed `reps`
        times: (ms per step, {family: ms per call}).  Small calls issued one
        by one from Python are bound by the host's launch rate; a graph
        replay measures the kernels."""
        import torch
        w = self.w

        def encodes():
            s = torch.cuda.current_stream()
            for l in range(w.layers):
                for r in range(2):
                    self.encode_call(l, r, self.x[l, r], s)

        def decodes():
            s = torch.cuda.current_stream()
            for l in range(w.layers):
                for r in range(2):
                    self.decode_call(l, r, s)

        out = {}
        for key, fn in (("step", self.step), ("enc", encodes), ("dec", decodes)):
            g = self.capture(fn)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                g.replay()
            b.record()
            torch.cuda.synchronize()
            out[key] = a.elapsed_time(b) / reps
            del g
        fam = "med3_encode" if w.med3 else "encode"
        return out["step"], {fam: out["enc"] / w.n_calls, "decode": out["dec"] / w.n_calls}


# DRAM bytes (read + write) of one hqmq_encode_med3 call of the 70B 128k call
# shape, from an ncu capture of its kernels, kept with the SHA-256 of the
# kernel sources it was taken on (profiles/traffic_encode_med3_call_llama3_70b_128k.md);
# a capture taken on other sources is reported as stale, not used.
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "traffic_encode_med3_call_llama3_70b_128k.md")
TRAFFIC_SHAPE = ((1, 8, 131072, 128), 32)


def kernel_sources_sha256():
    """SHA-256 over the CUDA sources of the library (file name and contents,
    in name order)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_quantization_hqmq_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def captured_traffic():
    """(bytes per call, note) from the traffic profile, or (None, why)."""
    try:
        text = open(TRAFFIC_PROFILE).read()
    except OSError:
        return None, "no traffic capture"
    vals = {}
    for line in text.splitlines():
        line = line.strip().lstrip("-* ").replace("`", "")
        if ":" in line and line.startswith(("traffic_bytes_per_call", "kernel_sources_sha256")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if "traffic_bytes_per_call" not in vals:
        return None, "no traffic figure in the capture summary"
    if vals.get("kernel_sources_sha256") != kernel_sources_sha256():
        return None, "stale: the kernel sources changed since the ncu capture"
    return int(vals["traffic_bytes_per_call"]), "ncu dram__bytes_read.sum + dram__bytes_write.sum of the call's kernels (profiles/)"


def one_read(w, table):
    """True when hqmq_encode_med3 reads x once: with search tables, since the
    bench runs Med3x in chunk mode."""
    return bool(w.med3 and table)


def algorithmic_bytes(w, n_outliers_per_call, table=True):
    """Bytes the method must move per call: x read once (twice when Med3x needs
    a second read), the codes (b/8 + 2 bytes per chunk) written, 12 bytes per
    outlier written (encode); codes and outliers read and bf16 y written
    (decode)."""
    B, H, T, D = w.call_shape
    n_chunks = B * H * T * D // 4
    x_bytes = B * H * T * D * w.elem_bytes
    b = math.ceil(math.log2(24 * w.S))
    code_bytes = n_chunks * (b / 8.0 + 2.0)
    out_bytes = n_outliers_per_call * 12.0 if w.med3 else 0.0
    return {
        # the scope's definition: with Med3x, x is read twice (the exact
        # median precedes classification), then the codes and the list
        "med3_encode": 2 * x_bytes + code_bytes + out_bytes,
        # what this implementation must move: in chunk mode with tables x is
        # read once (the encode runs before the median is known and only
        # possible outliers are revisited); element mode zeroes elements
        # before encoding and reads x twice
        "med3_encode_one_read": (1 if one_read(w, table) else 2) * x_bytes + code_bytes + out_bytes,
        "encode": x_bytes + code_bytes,
        "decode": code_bytes + out_bytes + B * H * T * D * 2,
    }


def alu_ops_per_chunk(S):
    """Lane operations of the S-codeword search per chunk:
    per secondary codeword one quaternion product (16 FMA), the 2T score
    (3 max + 3 add + 1 add + 1 max) and the argmax update (1 compare +
    2 select) = 27; per chunk ~60 more (load, norm, closed-form p, radius,
    packing)."""
    return 27 * S + 60


def kernel_stats(w, per_call_ms, peaks, n_out, table):
    """Per-call time and algorithmic HBM rate of each call family timed in
    `per_call_ms` {family: ms per call}."""
    ab = algorithmic_bytes(w, n_out, table)
    kern = {}
    for name in ("med3_encode", "encode", "decode"):
        if name not in per_call_ms:
            continue
        t = per_call_ms[name]
        gbs = ab[name] / (t * 1e-3) / 1e9
        kern[name] = {"ms_per_call": round(t, 4), "calls_per_step": w.n_calls,
                      "algorithmic_bytes_per_call": int(ab[name]),
                      "hbm_gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                      "bf16_gbs": round(w.call_elems * w.elem_bytes / (t * 1e-3) / 1e9, 1)}
        if name == "med3_encode":
            g1 = ab["med3_encode_one_read"] / (t * 1e-3) / 1e9
            kern[name]["one_read_bytes_per_call"] = int(ab["med3_encode_one_read"])
            kern[name]["one_read_hbm_frac"] = round(g1 / peaks["hbm_gbs"], 4)
    return kern


# the other workloads of the metric (S = 8 and S = 32), measured after the
# headline one: per call encode and decode rates
def run_attention(cache, peaks, iters=20, warmup=3):
    """Decode-phase attention read straight from the codes of layer 0 (one
    query token per sequence), timed with CUDA events; inputs (one layer's
    codes) are larger than L2.  Context: torch SDPA over the same layer
    decoded to dense bf16 (a library kernel)."""
    import torch
    import torch.nn.functional as F
    from kv_cache_quantization_hqmq_b200 import hqmq
    from kv_cache_quantization_hqmq_b200 import workloads as W
    w = cache.w
    B, H, T, D = w.call_shape
    Hq = w.n_q_heads
    if D != 128 or Hq % H or Hq // H > 8:
        return None
    dev = cache.x.device
    cbs, kv, dense, n_list = [], [], [], 0
    for r in range(2):
        cb = cache.codebook[r * H * w.S * 4:(r + 1) * H * w.S * 4]
        y = torch.empty(cache.shape, dtype=torch.bfloat16, device=dev)
        if w.med3:
            kv.append(hqmq.kv_codes(cache.words[0, r], cache.radius[0, r], cb, cache.out_idx[0, r],
                                    cache.out_val[0, r], cache.tile_off[0, r], cache.cap, cache.gran))
            hqmq.hqmq_decode(cache.words[0, r], cache.radius[0, r], cb, w.S, cache.out_idx[0, r],
                             cache.out_val[0, r], cache.slab_off[0, r], cache.cap, cache.gran, y,
                             tile_off=cache.tile_off[0, r])
            n_list += int(cache.slab_off[0, r][-1].item())
        else:
            kv.append(hqmq.kv_codes(cache.words[0, r], cache.radius[0, r], cb))
            hqmq.hqmq_decode(cache.words[0, r], cache.radius[0, r], cb, w.S, None, None, None, 0,
                             cache.gran, y)
        cbs.append(cb)
        dense.append(y)
    q = W.make_query(w, 0, device=dev)
    o = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    ws = hqmq.alloc_attention_ws(B, H, device=dev)
    st = hqmq.new_status(dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    ms = timed(lambda: hqmq.hqmq_attention_decode(q, kv[0], kv[1], w.S, H, T, o, ws, status=st))
    qd = q.view(B, Hq, 1, D)
    ms_dense = timed(lambda: F.scaled_dot_product_attention(qd, dense[0], dense[1], enable_gqa=True))

    def fake_quant():
        # the pipeline the pages compare against: decode both caches to dense
        # bf16 (this library's hqmq_decode), then attention over them
        for r in range(2):
            if w.med3:
                hqmq.hqmq_decode(cache.words[0, r], cache.radius[0, r], cbs[r], w.S,
                                 cache.out_idx[0, r], cache.out_val[0, r], cache.slab_off[0, r],
                                 cache.cap, cache.gran, dense[r], tile_off=cache.tile_off[0, r])
            else:
                hqmq.hqmq_decode(cache.words[0, r], cache.radius[0, r], cbs[r], w.S, None, None,
                                 None, 0, cache.gran, dense[r])
        F.scaled_dot_product_attention(qd, dense[0], dense[1], enable_gqa=True)
    ms_fake = timed(fake_quant)
    ref = F.scaled_dot_product_attention(qd, dense[0], dense[1], enable_gqa=True).float().view(B, Hq, D)
    b_idx = math.ceil(math.log2(24 * w.S))
    code_bytes = 2 * B * H * T * (4 * b_idx + 2 * D // 4) + n_list * (4 + 8)
    dense_bytes = 2 * B * H * T * D * 2
    gbs = code_bytes / (ms * 1e-3) / 1e9
    return {"op": "hqmq_attention_decode (k_attn)",
            "workload": "layer 0 of %s: batch %d, %d query heads over %d KV heads, %d tokens, S=%d"
                        % (w.name, B, Hq, H, T, w.S),
            "ms_per_call": round(ms, 4), "algorithmic_bytes": code_bytes,
            "gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
            "list_entries": n_list,
            "dense_bf16_sdpa_ms": round(ms_dense, 4),
            "dense_bf16_bytes": dense_bytes,
            "dense_over_hqmq_time": round(ms_dense / ms, 3),
            "decode_then_sdpa_ms": round(ms_fake, 4),
            "decode_then_sdpa_over_hqmq_time": round(ms_fake / ms, 3),
            "max_abs_diff_vs_sdpa": float((o - ref).abs().max().item()),
            "status_flags": hqmq.read_status(st)["flags"],
            "note": "dense_bf16_sdpa_ms: torch SDPA over caches already decoded (a library kernel); "
                    "decode_then_sdpa_ms: hqmq_decode of K and V to dense bf16, then that SDPA "
                    "(the decode-then-attend pipeline)"}


def run_qradius(cache, peaks, iters=20, warmup=3):
    """The quantized-radius variant on layer 0's K call (needs Med3x, chunk
    mode): hqmq_quantize_radius and hqmq_decode_qradius timed with CUDA
    events, bits per element, and the relative RMS error of both decodes
    against the input."""
    import torch
    from kv_cache_quantization_hqmq_b200 import hqmq
    w = cache.w
    if not w.med3:
        return None
    B, H, T, D = cache.shape
    dev = cache.x.device
    cb = cache.codebook[0:H * w.S * 4]
    rw = torch.empty(cache.n_words, dtype=torch.int32, device=dev)
    y = torch.empty(cache.shape, dtype=torch.bfloat16, device=dev)
    yq = torch.empty(cache.shape, dtype=torch.bfloat16, device=dev)
    st = hqmq.new_status(dev)
    args = (cache.words[0, 0], rw, cache.thr[0, 0], cb, w.S, cache.out_idx[0, 0],
            cache.out_val[0, 0], cache.tile_off[0, 0], cache.cap, cache.gran)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    ms_q = timed(lambda: hqmq.hqmq_quantize_radius(cache.radius[0, 0], cache.thr[0, 0],
                                                   cache.shape, w.S, rw))
    ms_d = timed(lambda: hqmq.hqmq_decode_qradius(*args, yq, st))
    hqmq.hqmq_decode(cache.words[0, 0], cache.radius[0, 0], cb, w.S, cache.out_idx[0, 0],
                     cache.out_val[0, 0], cache.slab_off[0, 0], cache.cap, cache.gran, y,
                     tile_off=cache.tile_off[0, 0])
    x = cache.x[0, 0].float()
    nx = x.norm()
    err_f16 = float((y.float() - x).norm() / nx)
    err_q = float((yq.float() - x).norm() / nx)
    n_chunks = cache.n_chunks
    b = math.ceil(math.log2(24 * w.S))
    n_out = int(cache.slab_off[0, 0][-1].item())
    q_bytes = n_chunks * (2 + b / 8)
    d_bytes = n_chunks * (2 * b / 8 + 8) + 12 * n_out
    # decode-phase attention over both caches in the quantized format
    att = None
    Hq = w.n_q_heads
    if D == 128 and Hq % H == 0 and Hq // H <= 8:
        from kv_cache_quantization_hqmq_b200 import workloads as W
        rwv = torch.empty(cache.n_words, dtype=torch.int32, device=dev)
        hqmq.hqmq_quantize_radius(cache.radius[0, 1], cache.thr[0, 1], cache.shape, w.S, rwv)
        kvs = [hqmq.kv_codes(cache.words[0, r], None, cache.codebook[r * H * w.S * 4:(r + 1) * H * w.S * 4],
                             cache.out_idx[0, r], cache.out_val[0, r], cache.tile_off[0, r], cache.cap,
                             cache.gran, rcode_words=(rw if r == 0 else rwv), thr=cache.thr[0, r])
               for r in range(2)]
        q = W.make_query(w, 0, device=dev)
        o = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
        aws = hqmq.alloc_attention_ws(B, H, device=dev)
        ms_a = timed(lambda: hqmq.hqmq_attention_decode(q, kvs[0], kvs[1], w.S, H, T, o, aws))
        n_list = n_out + int(cache.slab_off[0, 1][-1].item())
        a_bytes = 2 * B * H * T * (8 * b) + n_list * 12
        att = {"ms_per_call": round(ms_a, 4), "algorithmic_bytes": a_bytes,
               "hbm_frac": round(a_bytes / (ms_a * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    # the joint (index, level) block code and the 1-bit outlier flags
    joint = hqmq.alloc_joint(B, H, T, D, w.S, device=dev)
    flags = torch.empty(n_chunks // 32, dtype=torch.int32, device=dev)
    yj = torch.empty(cache.shape, dtype=torch.bfloat16, device=dev)
    ms_p = timed(lambda: hqmq.hqmq_pack_joint(cache.words[0, 0], rw, w.S, cache.shape, joint))
    ms_f = timed(lambda: hqmq.hqmq_list_flags(cache.out_idx[0, 0], cache.slab_off[0, 0], cache.cap,
                                              cache.shape, flags))
    ms_j = timed(lambda: hqmq.hqmq_decode_joint(joint, cache.thr[0, 0], cb, w.S, flags,
                                                cache.out_val[0, 0], cache.tile_off[0, 0],
                                                cache.cap, yj))
    hqmq.hqmq_decode_qradius(*args, yq, st)
    torch.cuda.synchronize()
    nblk, wbits = hqmq.hqmq_joint_block(w.S)
    n_el = B * H * T * D
    tiles = hqmq.hqmq_list_tiles(B, H, T, D)
    jb = {"codes": joint.numel() * 32 / n_el, "flags": n_chunks / n_el,
          "tile_offsets": (tiles + 1) * 32 / n_el, "values": n_out * 64 / n_el}
    jd_bytes = joint.numel() * 4 + n_chunks // 8 + n_out * 8 + n_el * 2
    joint_obj = {
        "chunks_per_block": nblk, "bits_per_block": wbits,
        "bits_per_element": {k: round(v, 4) for k, v in jb.items()},
        "bits_per_element_total": round(sum(jb.values()), 4),
        "pack_ms": round(ms_p, 4), "flags_ms": round(ms_f, 4), "decode_ms": round(ms_j, 4),
        "decode_hbm_frac": round(jd_bytes / (ms_j * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "decode_equals_qradius_decode": bool(torch.equal(yj.view(torch.int16), yq.view(torch.int16)))}
    return {"op": "hqmq_quantize_radius + hqmq_decode_qradius (layer 0, K)",
            "joint_code_with_flags": joint_obj,
            "attention_from_quantized_codes": att,
            "levels": 24 * w.S, "code_bits_per_chunk": 2 * b,
            "bits_per_element": round(2 * b / 4 + n_out * 96 / (B * H * T * D), 4),
            "bits_per_element_fp16_radius": round((b + 16) / 4 + n_out * 96 / (B * H * T * D), 4),
            "pages_bits_per_element": {"S8": 3.79, "S32": 5},
            "quantize_ms": round(ms_q, 4),
            "quantize_hbm_frac": round(q_bytes / (ms_q * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "decode_ms": round(ms_d, 4),
            "decode_hbm_frac": round(d_bytes / (ms_d * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "rel_rms_error": {"fp16_radius": round(err_f16, 5), "quantized_radius": round(err_q, 5)},
            "status_flags": hqmq.read_status(st)["flags"]}


def run_streaming(cache, iters=20, warmup=3):
    """One decode step of the whole model: for every (layer, role), the Med3x
    list of one new token per sequence under the prefill's threshold
    (hqmq_outlier_extract_given_thr) and its encode with that threshold, by
    the search table (hqmq_encode_lut) or the codeword loop (hqmq_encode),
    timed as plain launches and as one CUDA graph of the whole step.  The new
    tokens are drawn like the cache (same distribution, other seeds)."""
    import torch
    from kv_cache_quantization_hqmq_b200 import hqmq
    from kv_cache_quantization_hqmq_b200 import workloads as W
    w = cache.w
    if not w.med3:
        return None
    B, H, T, D = cache.shape
    dev = cache.x.device
    L2 = (w.layers, 2)
    wn = w.with_(input_seed=w.input_seed + 4242)
    x1 = torch.empty(L2 + (B, H, 1, D), dtype=w.torch_dtype, device=dev)
    for l in range(w.layers):
        for r in range(2):
            x1[l, r].copy_(W.make_call_input(wn, l, r, device=dev, tokens=1))
    n_words = hqmq.hqmq_index_words(B, H, 1, D, w.S)
    n_chunks = B * H * D // 4
    words = torch.empty(L2 + (n_words,), dtype=torch.int32, device=dev)
    radius = torch.empty(L2 + (n_chunks,), dtype=torch.int16, device=dev)
    oi = torch.empty(L2 + (n_chunks,), dtype=torch.int32, device=dev)
    ov = torch.empty(L2 + (4 * n_chunks,), dtype=torch.int16, device=dev)
    so = torch.empty(L2 + (B * H + 1,), dtype=torch.int32, device=dev)
    to = torch.empty(L2 + (hqmq.hqmq_list_tiles(B, H, 1, D) + 1,), dtype=torch.int32, device=dev)
    ws = torch.empty(L2 + (hqmq.hqmq_outlier_extract_given_thr_workspace_size(B, H, 1, D),),
                     dtype=torch.uint8, device=dev)

    def step(lut):
        for l in range(w.layers):
            for r in range(2):
                g0 = (l * 2 + r) * H
                cb = cache.codebook[g0 * w.S * 4:(g0 + H) * w.S * 4]
                hqmq.hqmq_outlier_extract_given_thr(x1[l, r], cache.thr[l, r], cache.gran, oi[l, r],
                                                    ov[l, r], so[l, r], n_chunks, ws[l, r],
                                                    tile_off=to[l, r])
                if lut:
                    tb = cache.table[g0 * cache.table_bytes:(g0 + H) * cache.table_bytes]
                    hqmq.hqmq_encode_lut(x1[l, r], cb, w.S, tb, cache.thr[l, r], cache.gran,
                                         words[l, r], radius[l, r])
                else:
                    hqmq.hqmq_encode(x1[l, r], cb, w.S, cache.thr[l, r], cache.gran, words[l, r],
                                     radius[l, r])

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    out = {"op": "decode-step append: hqmq_outlier_extract_given_thr + encode per (layer, role)",
           "new_tokens_per_step": B, "calls_per_step": w.layers * 2,
           "launches_per_step": 4 * w.layers * 2,
           "threshold": "per (layer, role, head) from the timed step (the prefill)"}
    for name, lut in (("search_table", True), ("codeword_loop", False)):
        if lut and cache.table is None:
            continue
        ms_plain = timed(lambda: step(lut))
        graph = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step(lut)
        torch.cuda.current_stream().wait_stream(s)
        with torch.cuda.graph(graph):
            step(lut)
        ms_graph = timed(graph.replay)
        out[name] = {"us_per_step_plain": round(ms_plain * 1e3, 1),
                     "us_per_step_graph": round(ms_graph * 1e3, 1)}
        del graph
    # all calls of the step in one launch (hqmq_append_batch), same outputs
    cbs = cache.codebook.view(w.layers * 2, H * w.S * 4)
    thr_all = cache.thr.view(w.layers * 2, H)
    oi_b = oi.view(-1)
    ov_b = ov.view(-1)
    xb = x1.view((w.layers * 2,) + x1.shape[2:])

    def batched():
        hqmq.hqmq_append_batch(xb, thr_all, cache.gran, cbs, w.S, words.view(-1), radius.view(-1),
                               oi_b, ov_b, so.view(-1), n_chunks, tile_off=to.view(-1))
    ms_plain = timed(batched)
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        batched()
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(graph):
        batched()
    ms_graph = timed(graph.replay)
    out["batched_one_launch"] = {"us_per_step_plain": round(ms_plain * 1e3, 1),
                                 "us_per_step_graph": round(ms_graph * 1e3, 1)}
    del graph
    out["outliers_last_step"] = int(so[:, :, -1].sum().item())
    return out


def run_covering(device, n_chunks=1 << 20):
    """The covering rate of the codebook measured with the GPU encode: mean and
    largest angle between a chunk and its decoded codeword over S = 1 .. 64 for
    Haar-random chunks (fp32), and the fitted slope of log mean angle against
    log 24 S (the pages' Proposition 3.1: -1/3)."""
    import torch
    from kv_cache_quantization_hqmq_b200 import hqmq
    g = torch.Generator(device=device)
    g.manual_seed(7)
    x = torch.randn((1, 1, n_chunks // 32, 128), generator=g, device=device)
    xu = torch.nn.functional.normalize(x.view(-1, 4), dim=1)
    out, Ss = {}, (1, 2, 4, 8, 16, 32, 64)
    means = []
    for S in Ss:
        cb = torch.empty(S * 4, dtype=torch.float32, device=device)
        hqmq.hqmq_make_codebook(11, S, 1, 0, cb)
        words, radius = hqmq.alloc_codes(1, 1, n_chunks // 32, 128, S, device=device)
        hqmq.hqmq_encode(x, cb, S, None, 0, words, radius)
        y = torch.empty_like(x)
        hqmq.hqmq_decode(words, radius, cb, S, None, None, None, 0, 0, y)
        yu = torch.nn.functional.normalize(y.view(-1, 4), dim=1)
        ang = torch.rad2deg(torch.arccos((xu * yu).sum(1).clamp(-1, 1)))
        means.append(float(ang.mean()))
        out["S%d" % S] = {"mean_deg": round(means[-1], 3), "max_deg": round(float(ang.max()), 3)}
    slope = float(np.polyfit(np.log(24.0 * np.array(Ss)), np.log(means), 1)[0])
    out["slope_log_mean_angle_vs_log_24S"] = round(slope, 4)
    out["chunks_per_S"] = n_chunks
    return out


SWEEP = ("llama3_8b", "qwen_outlier", "mha7b_s8", "mha7b_s32")


def run_sweep(device, peaks, steps=3, warmup=3, near_ties=None):
    import torch
    from kv_cache_quantization_hqmq_b200 import hqmq
    from kv_cache_quantization_hqmq_b200 import workloads as W
    out = {}
    for name in SWEEP:
        w = W.WORKLOADS[name]
        cache = Cache(w, 0, device)
        cache.setup()
        for _ in range(warmup):
            cache.step()
        torch.cuda.synchronize()
        st = hqmq.read_status(cache.status)
        # launches from Python (as the headline step) and the same work as
        # CUDA graphs (the device time of the kernels)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            cache.step()
        b.record()
        torch.cuda.synchronize()
        ms_plain = a.elapsed_time(b) / steps
        ms, per_call = cache.graph_times(steps)
        n_out = st["n_outliers"] / max(1, warmup) / w.n_calls if w.med3 else 0.0
        out[name] = {"S": w.S, "med3": ("chunk, C=%g" % w.C) if w.med3 else "off",
                     "cache_gb": round(w.cache_bytes / 1e9, 2), "ms_per_step": round(ms, 3),
                     "value_gbs": round(w.cache_bytes / (ms * 1e-3) / 1e9, 2),
                     "timing": "one CUDA graph per step (and per call family for the "
                               "kernels); ms_per_step_python_launches: the same step "
                               "launched call by call from Python",
                     "ms_per_step_python_launches": round(ms_plain, 3),
                     "kernels": kernel_stats(w, per_call, peaks, n_out, cache.table is not None),
                     "status_flags": st["flags"]}
        if near_ties is not None:
            near_ties[name] = oracle_parity_sample(cache, w.layers // 2, 1)
        del cache
        torch.cuda.empty_cache()
    return out


def run_hqmq(args):
    import torch
    rank, world, dist = dist_setup(args.gpus)
    device = torch.device("cuda", torch.cuda.current_device())
    from kv_cache_quantization_hqmq_b200 import hqmq
    from kv_cache_quantization_hqmq_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    peaks = load_peaks()

    # CPU baseline first, in spawned processes (no fork after CUDA init)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    cache = Cache(w, rank, device)
    setup_ms = cache.setup()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        cache.step()
    torch.cuda.synchronize()
    st = hqmq.read_status(cache.status)

    # each step is one CUDA graph of the step's launches (captured after the
    # warm-up), so that the host's launch rate does not enter the device time
    step_graph = cache.capture(cache.step)
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(dist)
    torch.cuda.synchronize()
    clocks.start()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        step_graph.replay()
    end.record()
    torch.cuda.synchronize()
    barrier(dist)
    clk = clocks.stop()
    ms_total = start.elapsed_time(end)
    ms_total = max_over_ranks(ms_total, dist, device)
    ms_step = ms_total / args.steps
    del step_graph

    # outside the timed region: the same step launched call by call from
    # Python, and the per-call times of the encode and decode calls (each
    # family of the step in one graph)
    a_ev = torch.cuda.Event(enable_timing=True)
    b_ev = torch.cuda.Event(enable_timing=True)
    a_ev.record()
    for _ in range(args.steps):
        cache.step()
    b_ev.record()
    torch.cuda.synchronize()
    ms_plain = a_ev.elapsed_time(b_ev) / args.steps
    _, per_call = cache.graph_times(args.steps)

    n_out = st["n_outliers"] / max(1, args.warmup) / w.n_calls if w.med3 else 0.0
    kern = kernel_stats(w, per_call, peaks, n_out, cache.table is not None)
    B, H, T, D = w.call_shape
    n_chunks = B * H * T * D // 4
    enc_key = "med3_encode" if w.med3 else "encode"
    t_enc = kern[enc_key]["ms_per_call"] * 1e-3
    alu_peak = ALU_LANES * peaks["sm_max_mhz"] * 1e6
    if cache.table is None and not w.med3:
        # the S-codeword loop: a fixed number of lane operations per chunk
        alu_achieved = alu_ops_per_chunk(w.S) * n_chunks / t_enc
        kern[enc_key]["alu_ops_per_chunk"] = alu_ops_per_chunk(w.S)
        kern[enc_key]["alu_frac"] = round(alu_achieved / alu_peak, 4)
        roof = {"kernel": "k_encode", "bound": "alu", "achieved": round(alu_achieved / 1e12, 3),
                "peak": round(alu_peak / 1e12, 3), "unit": "T lane-ops/s",
                "frac": round(alu_achieved / alu_peak, 4), "traffic": None,
                "peak_source": "148 SMs x 128 FP32 lanes x %s max SM MHz" % peaks["sm_max_mhz"]}
    else:
        if not w.med3:
            name = "k_encode_lut"
        elif one_read(w, cache.table is not None):
            name = ("hqmq_encode_med3 (one read of x: k_sample_window, k_encode_spec speculative "
                    "encode, k_finalize, k_list_fix)")
        else:
            name = "hqmq_encode_med3 (two reads of x: k_sample_window, k_pass_b, k_finalize, k_encode_lut)"
        roof = {"kernel": name, "bound": "hbm", "achieved": kern[enc_key]["hbm_gbs"],
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": kern[enc_key]["hbm_frac"],
                "traffic": None, "peak_source": peaks["source"]}
        if w.med3:
            roof["algorithmic_bytes"] = ("x read twice (the exact median precedes classification) + "
                                         "codes + 12 B per outlier, per call")
            roof["frac_one_read"] = kern[enc_key]["one_read_hbm_frac"]
            if (w.call_shape, w.S) == TRAFFIC_SHAPE and one_read(w, cache.table is not None):
                roof["traffic"], roof["traffic_source"] = captured_traffic()

    cache_bytes = w.cache_bytes
    value = world * cache_bytes / (ms_step * 1e-3) / 1e9
    b = math.ceil(math.log2(24 * w.S))
    bits = (b + 16) / 4.0
    n_elems_call = w.call_elems
    out_bits = (n_out * (64 + 32) / n_elems_call) if w.med3 else 0.0

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(cache, args, dist, device)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "kv_heads": H, "head_dim": D,
                   "batch": B, "tokens": T, "S": w.S, "med3": ("chunk, C=%g" % w.C) if w.med3 else "off",
                   "input": w.dtype, "cache_gb": round(cache_bytes / 1e9, 2),
                   "l2": "inputs larger than L2 (%.0f MB per call, %.1f GB per step)"
                         % (w.call_elems * w.elem_bytes / 1e6, cache_bytes / 1e9),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "value_is": "bf16 KV bytes through Med3x+encode+decode per second"},
        "kernels": kern,
        "encoder": "search table (exact)" if cache.table is not None else "S-codeword loop",
        "search_tables": None if cache.table is None else {
            "bytes_per_group": cache.table_bytes, "groups": w.n_groups,
            "bytes_per_call": cache.table_bytes * H, "total_bytes": cache.table_bytes * w.n_groups,
            "vs_cache_bytes": round(cache.table_bytes * w.n_groups / cache_bytes, 4)},
        "setup_ms": round(setup_ms, 3),
        "roofline": roof,
        "bits_per_element": {"ours_codes": bits, "ours_outliers": round(out_bits, 4),
                             "pages_S8": 3.79, "pages_S32": 5},
        "outlier_fraction": round(n_out / n_chunks, 5) if w.med3 else 0.0,
        "status_flags": st["flags"],
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": cache.kernels_per_step() * args.steps,
        "clocks": clk,
    }
    line["timing"] = ("each timed step is one CUDA graph replay of the step's launches; "
                      "ms_per_step_python_launches: the same step launched call by call from "
                      "Python; per-call kernel times from graphs of the step's encode calls and "
                      "of its decode calls")
    line["ms_per_step_python_launches"] = round(ms_plain, 3)
    if world == 1 and not args.no_cpu_baseline:
        line["near_ties"] = {w.name: oracle_parity_sample(cache, w.layers // 2, 1)}
    if world == 1 and not args.no_attention:
        line["attention"] = run_attention(cache, peaks)
        line["quantized_radius"] = run_qradius(cache, peaks)
        line["streaming_append"] = run_streaming(cache)
        line["covering"] = run_covering(device)
    if world == 1 and not args.no_sweep:
        # the metric's other workloads, after the headline's buffers are freed
        del cache
        torch.cuda.empty_cache()
        line["per_config"] = run_sweep(
            device, peaks, near_ties=line["near_ties"] if "near_ties" in line else None)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_e2e(cache, args, dist, device):
    """Same step through the C ABI with the input in pinned host memory: every
    call's input is copied H2D, and the compressed cache (index words, radii,
    the outlier list with its offsets) D2H, inside the timed region.
    Three streams: input copies (two device input buffers, so the copy of
    call i + 1 runs while call i is coded), the coding calls, and output
    copies.  The outlier lists are copied at their exact size: after the
    step's calls one D2H read of every call's list count, then one copy per
    call."""
    import torch
    w = cache.w
    call_bytes = w.call_elems * w.elem_bytes
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 16 << 30
    # distinct pinned host inputs (up to all calls, within half the free RAM)
    n_host = int(max(2, min(w.n_calls, (avail // 2) // (call_bytes + 1))))
    host_x = [torch.empty(cache.shape, dtype=w.torch_dtype, pin_memory=True) for _ in range(n_host)]
    for i, hx in enumerate(host_x):
        hx.copy_(cache.x[i // 2 % w.layers, i % 2])
    host_words = torch.empty(cache.n_words, dtype=torch.int32, pin_memory=True)
    host_rad = torch.empty(cache.n_chunks, dtype=torch.int16, pin_memory=True)
    if w.med3:
        host_oi = torch.empty(cache.cap, dtype=torch.int32, pin_memory=True)
        host_ov = torch.empty(cache.cap * 4, dtype=torch.int16, pin_memory=True)
        ns, nt = cache.slab_off.shape[-1], cache.tile_off.shape[-1]
        host_off = torch.empty(ns + nt, dtype=torch.int32, pin_memory=True)
        host_counts = torch.empty(w.n_calls, dtype=torch.int32, pin_memory=True)
    xbuf = [torch.empty(cache.shape, dtype=w.torch_dtype, device=device) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_run = torch.cuda.current_stream()
    moved = {"h2d": 0, "d2h": 0}

    def one_step():
        done = [None, None]              # per input buffer: its last call finished
        for i in range(w.n_calls):
            l, r = i // 2, i % 2
            k = i % 2
            if done[k] is not None:
                s_in.wait_event(done[k])
            with torch.cuda.stream(s_in):
                xbuf[k].copy_(host_x[i % n_host], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            moved["h2d"] += call_bytes
            s_run.wait_event(ready)
            cache.call(l, r, xbuf[k], s_run)
            fin = torch.cuda.Event()
            fin.record(s_run)
            done[k] = fin
            # the call's codes back to the host (one output buffer reused: the
            # copies are ordered on their stream)
            s_out.wait_event(fin)
            with torch.cuda.stream(s_out):
                host_words.copy_(cache.words[l, r], non_blocking=True)
                host_rad.copy_(cache.radius[l, r], non_blocking=True)
                if w.med3:
                    host_off[:ns].copy_(cache.slab_off[l, r], non_blocking=True)
                    host_off[ns:].copy_(cache.tile_off[l, r], non_blocking=True)
            moved["d2h"] += cache.n_words * 4 + cache.n_chunks * 2
            if w.med3:
                moved["d2h"] += (ns + nt) * 4
        if w.med3:
            # exact outlier lists: every call's count, then that many entries
            with torch.cuda.stream(s_out):
                s_out.wait_stream(s_run)
                host_counts.copy_(cache.slab_off[:, :, -1].reshape(-1), non_blocking=True)
            s_out.synchronize()
            moved["d2h"] += w.n_calls * 4
            for i, n in enumerate(host_counts.tolist()):
                n = max(0, min(int(n), cache.cap))
                l, r = i // 2, i % 2
                with torch.cuda.stream(s_out):
                    host_oi[:n].copy_(cache.out_idx[l, r, :n], non_blocking=True)
                    host_ov[:4 * n].copy_(cache.out_val[l, r, :4 * n], non_blocking=True)
                moved["d2h"] += n * 12
        s_run.wait_stream(s_out)
        s_run.wait_stream(s_in)

    steps = max(1, min(args.steps, 3))
    one_step()
    torch.cuda.synchronize()
    moved["h2d"] = moved["d2h"] = 0
    barrier(dist)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_run)
    s_in.wait_stream(s_run)
    for _ in range(steps):
        one_step()
    t1.record(s_run)
    torch.cuda.synchronize()
    barrier(dist)
    ms = max_over_ranks(t0.elapsed_time(t1), dist, device) / steps
    world = 1 if dist is None else dist.get_world_size()
    return {"value": round(world * w.cache_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 2), "steps": steps,
            "h2d_bytes_per_step": moved["h2d"] // steps, "d2h_bytes_per_step": moved["d2h"] // steps,
            "host_inputs": "%d distinct pinned call inputs reused round-robin" % n_host,
            "streams": "input copies, coding calls and output copies on three streams "
                       "(two device input buffers); outlier lists copied at their exact size"}


# ---------------------------------------------------------------- CPU oracle
def _oracle_sample_job(args):
    """Runs in a spawned process: the oracle's Med3x + encode + decode of one
    (head) slab sample of one call."""
    name, layer, role, tokens, head = args
    import numpy as np
    sys.path.insert(0, ROOT)
    from kv_cache_quantization_hqmq_b200 import workloads as W
    from oracle import hqmq_oracle as oracle
    w = W.WORKLOADS[name]
    x = W.as_numpy_bits(W.make_call_input(w, layer, role, tokens=tokens))
    x = np.ascontiguousarray(x[:, head:head + 1])
    B, H, T, D = x.shape
    g0 = W.group0(layer, role, w.heads) + head
    t0 = time.perf_counter()
    cb = oracle.make_codebook(w.codebook_seed, w.S, 1, g0)
    thr = None
    oi = ov = None
    if w.med3:
        rmed, thr = oracle.med3_threshold(x, w.C, 0)
        oi, ov, so, n, _ = oracle.extract(x, thr)
    words, rad, best, second, _ = oracle.encode(x, cb, w.S, thr=thr)
    oracle.decode(words, rad, cb, w.S, B, H, T, D, out_idx=oi, out_val=ov)
    return time.perf_counter() - t0, x.size * w.elem_bytes


def cpu_baseline(w, seconds_target=20.0):
    """The oracle, as it stands, on a bounded sample: the first `tokens`
    tokens of single-head slabs of layer 0, K and V, in parallel over the host
    cores (one spawned process per slab)."""
    import multiprocessing as mp
    cores = os.cpu_count() or 1
    # calibrate: brute force costs ~24 S codewords per chunk
    probe_tokens = 256
    ctx = mp.get_context("spawn")
    with ctx.Pool(1) as pool:
        t, nbytes = pool.map(_oracle_sample_job, [(w.name, 0, 0, probe_tokens, 0)])[0]
    per_token = t / probe_tokens
    n_jobs = min(cores, 2 * w.heads)
    tokens = int(max(probe_tokens, min(w.tokens, seconds_target / max(per_token, 1e-9))))
    tokens = max(32, (tokens // 32) * 32)
    jobs = [(w.name, 0, j % 2, tokens, (j // 2) % w.heads) for j in range(n_jobs)]
    t0 = time.perf_counter()
    with ctx.Pool(n_jobs) as pool:
        res = pool.map(_oracle_sample_job, jobs)
    wall = time.perf_counter() - t0
    total_bytes = sum(r[1] for r in res)
    busy = max(r[0] for r in res)
    return {"value": round(total_bytes / busy / 1e9, 6), "unit": "GB/s", "cores": n_jobs,
            "kind": "oracle",
            "sample": "%d single-head slabs (layer 0, K and V) x %d tokens x batch %d of %s; "
                      "Med3x + encode + decode by the plain C oracle, one process per slab; "
                      "wall %.1f s" % (n_jobs, tokens, w.batch, w.name, wall)}


NEAR_TIE_REL = 1e-6


def oracle_parity_sample(cache, layer, role, n_sample=8192, seed=0):
    """Part of the oracle (cpu_baseline) leg, after the timed region: the
    GPU's codes of one benched call (the last step's) against the CPU oracle
    on the same input bytes.  Med3x threshold and the whole ordered outlier
    list are compared in full; indices and radii on a seeded sample of
    chunks.  An index that differs is exempt only if the oracle's fp32 score
    of the GPU's pick is within 1e-6 (relative) of its best score; such
    near-ties are counted, anything else is reported as non-exempt."""
    import torch
    from kv_cache_quantization_hqmq_b200 import workloads as W
    from oracle import hqmq_oracle as oracle
    w = cache.w
    B, H, T, D = cache.shape
    torch.cuda.synchronize()
    x = W.as_numpy_bits(cache.x[layer, role])
    g0 = W.group0(layer, role, H)
    cb = oracle.make_codebook(w.codebook_seed, w.S, H, g0)
    cb_gpu = cache.codebook[g0 * w.S * 4:(g0 + H) * w.S * 4].cpu().numpy()
    out = {"call": "layer %d, role %s" % (layer, "KV"[role]),
           "codebook_bits_equal": bool(np.array_equal(cb.reshape(-1).view(np.uint32),
                                                      cb_gpu.view(np.uint32)))}
    thr = None
    if w.med3:
        _, thr = oracle.med3_threshold(x, w.C, 0)
        thr_g = cache.thr[layer, role].cpu().numpy()
        out["thr_bits_equal"] = bool(np.array_equal(thr.view(np.uint32), thr_g.view(np.uint32)))
        idx_o, val_o, so_o, n_o, _ = oracle.extract(x, thr, cap=cache.cap)
        so_g = cache.slab_off[layer, role].cpu().numpy().view(np.uint32)
        k = min(n_o, cache.cap)
        oi_g = cache.out_idx[layer, role][:k].cpu().numpy().view(np.uint32)
        ov_g = cache.out_val[layer, role][:4 * k].cpu().numpy().view(np.uint16).reshape(-1, 4)
        out["list_entries"] = int(n_o)
        out["list_bits_equal"] = bool(np.array_equal(so_g, so_o) and np.array_equal(oi_g, idx_o[:k])
                                      and np.array_equal(ov_g, val_o[:k].reshape(-1, 4)))
    rng = np.random.default_rng(seed + 1000 * layer + role)
    chunks = np.sort(rng.choice(cache.n_chunks, min(n_sample, cache.n_chunks), replace=False))
    chunks = chunks.astype(np.int64)
    idx_o, rad_o, best, second = oracle.encode_chunks(x, cb, w.S, chunks, thr=thr)
    words_g = cache.words[layer, role].cpu().numpy().view(np.uint32)
    idx_g = oracle.get_index(words_g, w.S, chunks)
    rad_g = cache.radius[layer, role].cpu().numpy().view(np.uint16)[chunks]
    mm = np.nonzero(idx_g != idx_o)[0]
    exempt = 0
    if mm.size:
        sg = oracle.score_chunks(x, cb, w.S, chunks[mm], idx_g[mm], thr=thr)
        gap = best[mm].astype(np.float64) - sg.astype(np.float64)
        exempt = int(np.sum(gap <= NEAR_TIE_REL * np.abs(best[mm].astype(np.float64))))
    near = int(np.sum((best > 0) & (best.astype(np.float64) - second.astype(np.float64)
                                    <= NEAR_TIE_REL * np.abs(best.astype(np.float64)))))
    out.update({"checked_chunks": int(chunks.size), "index_mismatches": int(mm.size),
                "mismatched_exempt": exempt, "mismatched_not_exempt": int(mm.size) - exempt,
                "radius_mismatches": int(np.sum(rad_g != rad_o)),
                "near_tie_pairs_in_sample": near})
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from kv_cache_quantization_hqmq_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    times = []
    cpu = None
    per_step = max(3.0, 60.0 / max(1, args.steps + args.warmup))
    if args.ref_seconds is not None:
        per_step = args.ref_seconds
    for i in range(args.warmup + args.steps):
        cpu = cpu_baseline(w, per_step)
        if i >= args.warmup:
            times.append(cpu["value"])
    value = statistics.mean(times)
    cpu["value"] = round(value, 6)
    line = {"metric": METRIC, "value": round(value, 6), "unit": "GB/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)), "steps": args.steps,
            "warmup": args.warmup,
            # a whole step's bf16 cache bytes at the sample's rate
            "ms_per_step": round(w.cache_bytes / (value * 1e9) * 1e3, 1),
            "ms_per_step_is": "extrapolated: the step's cache bytes at the rate of the timed sample",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "S": w.S,
                       "med3": ("chunk, C=%g" % w.C) if w.med3 else "off"},
            "impl": "reference", "cpu_baseline": cpu,
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="hqmq", choices=["hqmq", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-config encode/decode rates of the other workloads")
    ap.add_argument("--no-attention", action="store_true",
                    help="skip the decode-phase attention measurement on layer 0's codes")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="oracle seconds per step of --impl reference (default: about "
                         "60 s over all steps)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_hqmq(args)


if __name__ == "__main__":
    main()
