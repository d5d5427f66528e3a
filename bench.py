#!/usr/bin/env python3
"""Benchmark of the exact attention path on B200: one JSON line per run.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl ours|reference]

A step is one call of the library on one batch of synthetic input (iid N(0,1), seeded,
counter-based generator in ``synth``), with the inputs resident in HBM.  The headline workload
is the largest single-GPU prefill: causal sliding-window attention, B=1, Hq=32, Hkv=8 (GQA),
n=32768, d=128, a 4096-key window plus 4 always-visible sink tokens, bf16 (fp32 accumulate).
The same line carries, each with its own timing, roofline, end-to-end figure, clocks and CPU
baseline, the GQA causal prefill (B=2, Hq=32, Hkv=8, n=8192) under "gqa_causal", the causal
prefill (B=4, Hq=Hkv=16, n=2048) under "causal", and the split-K decode workload (64 sequences x
1 token, Hq=32, Hkv=8, 32768 cached keys) under "decode", because the metric names both prefill
and decode.

Timing: W warm-up steps, then K timed steps; before every timed step a 256 MiB buffer is
written (more than the 126 MB L2) and the step itself is bracketed by CUDA events on the
launching stream; ``ms_per_step`` is the mean of the K event intervals.  The headline and the
decode entry time exactly K steps; the two other prefill entries time at least K steps and as
many more as give about 0.2 s of device time, so that the clock sampler (NVML, every 1 ms) sees
the GPU under load; their own ``steps`` says how many.  With N > 1 (torchrun,
one process per GPU) every rank runs its own replica of the workload on its own GPU (weak
scaling: independent batches, no data-path collective), the ranks meet at a barrier before and
after the timed loop, and the slowest rank's time sets the whole-job throughput.

``--impl reference`` times the fp64 CPU oracle (the repository's reference implementation of
the same operation) on bounded samples of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s & % BF16 TC peak (prefill); decode HBM GB/s & % peak"
FULL, CAUSAL, SLIDING, LOCAL_GLOBAL = 0, 1, 2, 3
MASK_NAMES = {FULL: "full", CAUSAL: "causal", SLIDING: "sliding", LOCAL_GLOBAL: "local+global"}

WORKLOADS = {
    "full_b1_h1_n256_d64_f32": dict(kind="fwd_f32", B=1, Hq=1, Hkv=1, N=256, d=64, mask=FULL,
                                    window=0, n_sink=0, seed=1),
    "causal_b4_h16_n2048_d128": dict(kind="fwd", B=4, Hq=16, Hkv=16, N=2048, d=128,
                                     mask=CAUSAL, window=0, n_sink=0, seed=2),
    "gqa_causal_b2_h32_kv8_n8192_d128": dict(kind="fwd", B=2, Hq=32, Hkv=8, N=8192, d=128,
                                             mask=CAUSAL, window=0, n_sink=0, seed=3),
    "sliding_b1_h32_kv8_n32768_w4096_s4_d128": dict(kind="fwd", B=1, Hq=32, Hkv=8, N=32768,
                                                    d=128, mask=SLIDING, window=4096, n_sink=4,
                                                    seed=4),
    "decode_b64_h32_kv8_n32768_d128": dict(kind="decode", B=64, Hq=32, Hkv=8, N=32768, d=128,
                                           mask=FULL, window=0, n_sink=0, seed=5),
    # 16 packed sequences of mixed lengths (32,768 tokens), causal, cu_seqlens form
    "varlen_causal_16seq_32k_h16_d128": dict(kind="fwd_varlen", B=16, Hq=16, Hkv=16, N=32768,
                                             d=128, mask=CAUSAL, window=0, n_sink=0, seed=6,
                                             lens=[4096, 3584, 3072, 2816, 2560, 2304, 2048, 1792,
                                                   1664, 1536, 1536, 1280, 1280, 1024, 1024, 1152]),
    # bidirectional (Longformer) window of 2048 keys on each side + 4 global tokens
    "local_global_b1_h32_kv8_n32768_w2048_g4_d128": dict(kind="fwd", B=1, Hq=32, Hkv=8, N=32768,
                                                         d=128, mask=LOCAL_GLOBAL, window=2048,
                                                         n_sink=4, seed=9),
    # the headline workload with E4M3 (FP8) Q, K, V and per-(b, head) scales
    "fp8_causal_b4_h16_n2048_d128": dict(kind="fwd_fp8", B=4, Hq=16, Hkv=16, N=2048, d=128,
                                         mask=CAUSAL, window=0, n_sink=0, seed=10),
    # backward pass of the headline workload (dQ, dK, dV from the forward's O and LSE)
    "bwd_causal_b4_h16_n2048_d128": dict(kind="bwd", B=4, Hq=16, Hkv=16, N=2048, d=128,
                                         mask=CAUSAL, window=0, n_sink=0, seed=8),
    # the decode workload over a paged cache: 16-token pages in a seeded random order
    "paged_decode_b64_h32_kv8_n32768_p16_d128": dict(kind="decode_paged", B=64, Hq=32, Hkv=8,
                                                     N=32768, d=128, mask=FULL, window=0,
                                                     n_sink=0, seed=7, page_size=16),
    # a fixed block-sparse layout (BigBird style: diagonal band, global first block row and
    # column, 3 random blocks per row) over a full base mask
    "block_sparse_b1_h32_kv8_n32768_d128": dict(kind="fwd_block_sparse", B=1, Hq=32, Hkv=8,
                                                N=32768, d=128, mask=FULL, window=0, n_sink=0,
                                                seed=11, n_random=3),
    # an eighth of the decode workloads (1 GiB of cache), for ncu captures that must stay small
    "decode_b8_h32_kv8_n32768_d128": dict(kind="decode", B=8, Hq=32, Hkv=8, N=32768, d=128,
                                          mask=FULL, window=0, n_sink=0, seed=5),
    "paged_decode_b8_h32_kv8_n32768_p16_d128": dict(kind="decode_paged", B=8, Hq=32, Hkv=8,
                                                    N=32768, d=128, mask=FULL, window=0,
                                                    n_sink=0, seed=7, page_size=16),
}
PROFILING_ONLY = ("decode_b8_h32_kv8_n32768_d128", "paged_decode_b8_h32_kv8_n32768_p16_d128")
# fp32 FMA peak of the CUDA cores (TFLOP/s), for the fp32 workload, which uses no tensor core
FP32_FMA_PEAK_TFLOPS = round(148 * 128 * 2 * 1965e6 / 1e12, 1)
HEADLINE = "sliding_b1_h32_kv8_n32768_w4096_s4_d128"
DECODE = "decode_b64_h32_kv8_n32768_d128"
# entries of the default line besides the headline: (key, workload, fixed step count?)
EXTRAS = (("gqa_causal", "gqa_causal_b2_h32_kv8_n8192_d128", False),
          ("causal", "causal_b4_h16_n2048_d128", False),
          ("decode", DECODE, True))
# nominal datasheet denominators, quoted beside the measured ones: dense bf16 tensor peak of a
# B200, and the HBM bandwidth the decode target is stated against
NOMINAL = {"tensor": 2250.0, "hbm": 8000.0}
MIN_TIMED_MS = 200.0

# DRAM traffic per launch of each workload's dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the hash of the sources of that
# kernel family (kernel_sources_hash); reported as null once those sources differ.
NCU_TRAFFIC = {
    "full_b1_h1_n256_d64_f32": {"bytes": 260608, "src": "02e210e28044d0c4"},
    "causal_b4_h16_n2048_d128": {"bytes": 130977024, "src": "e769cf1b4f770bb4"},
    "gqa_causal_b2_h32_kv8_n8192_d128": {"bytes": 499211008, "src": "e769cf1b4f770bb4"},
    "sliding_b1_h32_kv8_n32768_w4096_s4_d128": {"bytes": 703764224, "src": "e769cf1b4f770bb4"},
    "varlen_causal_16seq_32k_h16_d128": {"bytes": 1233493784, "src": "e769cf1b4f770bb4"},
    "local_global_b1_h32_kv8_n32768_w2048_g4_d128": {"bytes": 758468096, "src": "e769cf1b4f770bb4"},
    "fp8_causal_b4_h16_n2048_d128": {"bytes": 54257408, "src": "e769cf1b4f770bb4"},
    "block_sparse_b1_h32_kv8_n32768_d128": {"bytes": 913352960, "src": "e769cf1b4f770bb4"},
    # the backward step's three kernels together (prep + dK/dV + dQ)
    "bwd_causal_b4_h16_n2048_d128": {"bytes": 1042068480, "src": "d33920bcb6ed5264"},
    # a decode step's two kernels together (split + combine), captured on the 8-sequence
    # cases; the cache is read once per sequence, so the 64-sequence step moves 8x that
    "decode_b64_h32_kv8_n32768_d128": {"bytes": 8 * 1084886016, "src": "1a9ec2fd52b8d638"},
    "decode_b8_h32_kv8_n32768_d128": {"bytes": 1084886016, "src": "1a9ec2fd52b8d638"},
    "paged_decode_b64_h32_kv8_n32768_p16_d128": {"bytes": 8 * 1085015520, "src": "1a9ec2fd52b8d638"},
    "paged_decode_b8_h32_kv8_n32768_p16_d128": {"bytes": 1085015520, "src": "1a9ec2fd52b8d638"},
}

# the device sources each kernel family is compiled from (the launch code in abi.cu only sets
# up grids and tensor maps)
FAMILY_SOURCES = {
    "prefill": ("fwd_sm100.cuh", "common.cuh", "dev/ptx.cuh", "dev/ptx_f8.cuh", "dev/ptx_store.cuh"),
    "decode": ("decode.cuh", "decode_tc.cuh", "common.cuh", "dev/ptx.cuh", "dev/ptx_store.cuh"),
    "bwd": ("bwd_sm100.cuh", "common.cuh", "dev/ptx.cuh", "dev/ptx_store.cuh"),
    "f32": ("fwd_f32.cuh", "common.cuh"),
}


def family_of(w):
    if w["kind"] in ("decode", "decode_paged"):
        return "decode"
    if w["kind"] == "fwd_f32":
        return "f32"
    return "bwd" if w["kind"] == "bwd" else "prefill"


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def code_tokens(text: str) -> str:
    """Source text without comments and with runs of white space collapsed: edits to comments
    or layout do not change what the compiler builds, so they keep the hash."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_sources_hash(family: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_82_b200", "csrc")
    for f in FAMILY_SOURCES[family]:
        with open(os.path.join(csrc, f)) as fh:
            h.update((f + "\0" + code_tokens(fh.read())).encode())
    return h.hexdigest()[:16]


def fp8_gemm_peak():
    """Measured dense E4M3 tensor throughput of this GPU (TFLOP/s): torch._scaled_mm (cuBLASLt)
    on 8192^3 E4M3 x E4M3 -> bf16 with per-tensor scales, best of 10 after 3 warm-ups (the
    method the bf16 figure of MEASURED_PEAKS.json uses, with the FP8 GEMM).  None if the call is
    unavailable."""
    import torch

    n = 8192
    try:
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()  # column-major
        one = torch.ones((), device="cuda")
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return round(2 * n ** 3 / (best * 1e-3) / 1e12, 1)
    except (RuntimeError, AttributeError, TypeError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------------------------
# work accounting
# ----------------------------------------------------------------------------------------------
def work_of(w):
    from exact_io_aware_82_b200 import accounting as acc

    if w["kind"] == "decode":
        return acc.decode_bytes(w["B"], w["Hq"], w["Hkv"], w["N"], w["d"]), "GB/s", 1e9
    if w["kind"] == "decode_paged":
        return acc.decode_paged_bytes(w["B"], w["Hq"], w["Hkv"], w["N"], w["d"], w["page_size"]), \
            "GB/s", 1e9
    if w["kind"] == "fwd_varlen":
        fl = sum(acc.attn_flops(1, w["Hq"], n, n, w["d"], w["mask"], w["window"], w["n_sink"])
                 for n in w["lens"])
        return fl, "TFLOP/s", 1e12
    if w["kind"] == "fwd_block_sparse":
        import synth

        nt = -(-w["N"] // 128)
        bm = synth.block_layout_bigbird(w["seed"], nt, nt, w["n_random"])
        pairs = acc.block_sparse_pairs(bm, w["N"], w["N"], w["mask"], w["window"], w["n_sink"],
                                       Hq=w["Hq"])
        return 4 * w["d"] * w["B"] * pairs, "TFLOP/s", 1e12
    if w["kind"] == "bwd":
        return acc.attn_bwd_flops(w["B"], w["Hq"], w["N"], w["N"], w["d"], w["mask"], w["window"],
                                  w["n_sink"]), "TFLOP/s", 1e12
    fl = acc.attn_flops(w["B"], w["Hq"], w["N"], w["N"], w["d"], w["mask"], w["window"],
                        w["n_sink"])
    return fl, "TFLOP/s", 1e12


def config_of(name, w, n_gpus):
    c = {"workload": name, "B": w["B"], "Hq": w["Hq"], "Hkv": w["Hkv"], "d": w["d"],
         "mask": MASK_NAMES[w["mask"]]}
    if w["kind"] in ("decode", "decode_paged"):
        c.update({"q_tokens": 1, "kv_len": w["N"]})
    if w["kind"] == "decode_paged":
        c.update({"page_size": w["page_size"], "page_order": "seeded random permutation"})
    elif w["kind"] == "fwd_varlen":
        c.update({"num_seqs": len(w["lens"]), "total_tokens": sum(w["lens"]), "seq_lens": w["lens"]})
    else:
        c.update({"n": w["N"]})
    if w["mask"] == SLIDING:
        c.update({"window": w["window"], "n_sink": w["n_sink"]})
    if w["mask"] == LOCAL_GLOBAL:
        c.update({"window_each_side": w["window"], "n_global": w["n_sink"]})
    if w["kind"] == "fwd_block_sparse":
        c.update({"layout": "128x128 blocks: diagonal band of 3, first block row and column, "
                            "%d seeded random blocks per row; one layout for all heads" % w["n_random"]})
    c["inputs"] = {"fwd_f32": "fp32", "fwd_fp8": "e4m3 codes, fp32 scale per (b, head)"}.get(
        w["kind"], "bf16")
    c["l2"] = "flushed before every timed step (256 MiB write)"
    c["parallelism"] = "replicas x%d (independent batch per GPU, no collective)" % n_gpus
    return c


# ----------------------------------------------------------------------------------------------
# clock sampling (NVML, read-only) during the timed region
# ----------------------------------------------------------------------------------------------
_REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index, interval_s=0.001):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval_s
        self.ok = False
        try:
            import pynvml

            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = h
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.err = repr(e)
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                bits = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, n in _REASON_BITS.items():
                    if bits & b:
                        self.reasons.add(n)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------------------------
class Workload:
    """Device buffers and the step function of one workload on the current GPU.  ``inputs`` lists
    every tensor a step reads (the end-to-end timing copies each of them from the host)."""

    def __init__(self, name, rank):
        import torch

        import synth
        from exact_io_aware_82_b200 import attn as A

        self.name, self.w = name, WORKLOADS[name]
        w = self.w
        self.A = A
        seed = rank_seed(w["seed"], rank)
        dt = torch.float32 if w["kind"] == "fwd_f32" else torch.bfloat16
        B, Hq, Hkv, N, d = w["B"], w["Hq"], w["Hkv"], w["N"], w["d"]
        self.ws = None
        self.lse = None
        self.launches_per_step = 1
        if w["kind"] == "fwd_varlen":
            # packed token-major tensors and the per-sequence offsets
            total = sum(w["lens"])
            assert total == N
            q = synth.normal_torch(seed, synth.Q_ID, (total, Hq, d), dt, "cuda")
            k = synth.normal_torch(seed, synth.K_ID, (total, Hkv, d), dt, "cuda")
            v = synth.normal_torch(seed, synth.V_ID, (total, Hkv, d), dt, "cuda")
            cu = torch.tensor(np_cumsum0(w["lens"]), dtype=torch.int32, device="cuda")
            self.inputs = [q, k, v, cu]
            self.lse = torch.empty((total, Hq), dtype=torch.float32, device="cuda")
            self.max_len = max(w["lens"])
        elif w["kind"] == "decode_paged":
            ps = w["page_size"]
            table = paged_table(w)
            num_pages = table.size
            q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, 1, d), dt, "cuda")
            k = synth.normal_torch(seed, synth.K_ID, (num_pages, ps, Hkv, d), dt, "cuda")
            v = synth.normal_torch(seed, synth.V_ID, (num_pages, ps, Hkv, d), dt, "cuda")
            bt = torch.from_numpy(table).cuda()
            sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
            self.inputs = [q, k, v, bt, sl]
            self.lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        elif w["kind"] == "fwd_fp8":
            # E4M3 codes with per-(b, head) scales, drawn on the host
            xs, scs = [], []
            for tid, shape in ((synth.Q_ID, (B, Hq, N, d)), (synth.K_ID, (B, Hkv, N, d)),
                               (synth.V_ID, (B, Hkv, N, d))):
                codes, sc = synth.normal_e4m3(seed, tid, shape)
                xs.append(torch.from_numpy(codes).cuda())
                scs.append(torch.from_numpy(sc).cuda())
            self.inputs = xs + scs
            self.lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
            self.o = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device="cuda")
        elif w["kind"] == "fwd_block_sparse":
            q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, N, d), dt, "cuda")
            k = synth.normal_torch(seed, synth.K_ID, (B, Hkv, N, d), dt, "cuda")
            v = synth.normal_torch(seed, synth.V_ID, (B, Hkv, N, d), dt, "cuda")
            nt = -(-N // 128)
            bm = torch.from_numpy(synth.block_layout_bigbird(w["seed"], nt, nt, w["n_random"])).cuda()
            self.inputs = [q, k, v, bm]
            self.lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
        elif w["kind"] == "bwd":
            # the forward's outputs for these inputs are inputs of the backward step
            q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, N, d), dt, "cuda")
            k = synth.normal_torch(seed, synth.K_ID, (B, Hkv, N, d), dt, "cuda")
            v = synth.normal_torch(seed, synth.V_ID, (B, Hkv, N, d), dt, "cuda")
            dout = synth.normal_torch(seed, synth.DO_ID, (B, Hq, N, d), dt, "cuda")
            o, lse = A.attn_fwd(q, k, v, mask_kind=w["mask"], window=w["window"],
                                n_sink=w["n_sink"])
            self.inputs = [q, k, v, o, lse, dout]
            self.grads = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
            self.ws = torch.empty(A.attn_bwd_workspace_bytes(B, Hq, N, N, w["mask"], w["window"],
                                                             w["n_sink"]), dtype=torch.uint8,
                                  device="cuda")
            self.launches_per_step = 3
        else:
            nq = 1 if w["kind"] == "decode" else N
            q = synth.normal_torch(seed, synth.Q_ID, (B, Hq, nq, d), dt, "cuda")
            k = synth.normal_torch(seed, synth.K_ID, (B, Hkv, N, d), dt, "cuda")
            v = synth.normal_torch(seed, synth.V_ID, (B, Hkv, N, d), dt, "cuda")
            self.inputs = [q, k, v]
            lse_shape = (B, Hq) if w["kind"] == "decode" else (B, Hq, nq)
            self.lse = torch.empty(lse_shape, dtype=torch.float32, device="cuda")
        if w["kind"] != "fwd_fp8":
            self.o = torch.empty_like(self.inputs[0])
        # what a step hands back to its caller (read back in the end-to-end timing)
        self.outputs = self.grads if w["kind"] == "bwd" else [self.o, self.lse]
        if w["kind"] in ("decode", "decode_paged"):
            nb = A.attn_decode_workspace_bytes(B, Hq, Hkv, N, d, 0)
            self.ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
            self.launches_per_step = 2

    def run(self, inputs=None):
        w, A = self.w, self.A
        x = self.inputs if inputs is None else inputs
        o, lse = self.o, self.lse
        if w["kind"] == "decode":
            A.attn_decode(x[0], x[1], x[2], o=o, lse=lse, workspace=self.ws)
        elif w["kind"] == "fwd_fp8":
            A.attn_fwd_fp8(x[0], x[1], x[2], x[3], x[4], x[5], o=o, lse=lse, mask_kind=w["mask"],
                           window=w["window"], n_sink=w["n_sink"])
        elif w["kind"] == "bwd":
            g = self.grads
            A.attn_bwd(x[0], x[1], x[2], x[3], x[4], x[5], mask_kind=w["mask"], window=w["window"],
                       n_sink=w["n_sink"], dq=g[0], dk=g[1], dv=g[2], workspace=self.ws)
        elif w["kind"] == "decode_paged":
            A.attn_decode_paged(x[0], x[1], x[2], x[3], x[4], w["N"], o=o, lse=lse,
                                workspace=self.ws)
        elif w["kind"] == "fwd_varlen":
            A.attn_fwd_varlen(x[0], x[1], x[2], x[3], x[3], self.max_len, o=o, lse=lse,
                              mask_kind=w["mask"], window=w["window"], n_sink=w["n_sink"])
        elif w["kind"] == "fwd_block_sparse":
            A.attn_fwd_block_sparse(x[0], x[1], x[2], x[3], o=o, lse=lse, mask_kind=w["mask"],
                                    window=w["window"], n_sink=w["n_sink"])
        elif w["kind"] == "fwd_f32":
            A.attn_fwd_f32(x[0], x[1], x[2], o=o, lse=lse, mask_kind=w["mask"],
                           window=w["window"], n_sink=w["n_sink"])
        else:
            A.attn_fwd(x[0], x[1], x[2], o=o, lse=lse, mask_kind=w["mask"], window=w["window"],
                       n_sink=w["n_sink"])


def np_cumsum0(lens):
    out = [0]
    for n in lens:
        out.append(out[-1] + n)
    return out


def paged_table(w):
    """Block table [B][N / page_size] of a paged workload: every page of the pool used once, in
    a seeded random order (the same on every rank and for the oracle sample)."""
    import numpy as np

    per_seq = w["N"] // w["page_size"]
    perm = np.random.default_rng(w["seed"]).permutation(w["B"] * per_seq).astype(np.int32)
    return perm.reshape(w["B"], per_seq)


def timed_loop(fn, steps, warmup, flush, dist_on, sampler=None):
    """W warm-ups, then K steps each bracketed by CUDA events, with an L2 flush before each."""
    import torch

    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    if dist_on:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        for s, e in ev:
            flush.zero_()
            s.record(stream)
            fn()
            e.record(stream)
        torch.cuda.synchronize()
    if dist_on:
        import torch.distributed as dist

        dist.barrier()
    return [s.elapsed_time(e) for s, e in ev]


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling): seed offset by the rank."""
    return base_seed + 1000 * rank


def max_over_ranks(x, dist_on, device="cuda"):
    """The slowest rank's value (timing is reported as the max over ranks)."""
    if not dist_on:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(work_per_step, steps, total_ms_max, world, scale):
    """Aggregate throughput of all ranks: every rank did work_per_step x steps in at most
    total_ms_max milliseconds."""
    return world * work_per_step * steps / (total_ms_max * 1e-3) / scale


def measure_ours(name, steps, warmup, rank, world, dist_on, flush, peaks, peak_kind,
                 min_timed_ms=0.0):
    """Time one workload.  With min_timed_ms > 0 the step count grows past ``steps`` until the
    timed steps add up to about that much device time (the same count on every rank)."""
    import torch

    wl = Workload(name, rank)
    w = wl.w
    work, unit, scale = work_of(w)
    A = wl.A
    if min_timed_ms > 0:
        probe = timed_loop(wl.run, 3, warmup, flush, dist_on)
        est = max_over_ranks(min(probe), dist_on)
        steps = max(steps, int(math.ceil(min_timed_ms / max(est, 1e-3))))
    sampler = ClockSampler(torch.cuda.current_device())
    times = timed_loop(wl.run, steps, warmup, flush, dist_on, sampler)
    err = A.attn_get_device_error()
    if err != 0:
        raise RuntimeError("device error flag set after the timed loop: %d" % err)
    total_ms = max_over_ranks(sum(times), dist_on)
    ms_per_step = total_ms / steps
    value = whole_job_value(work, steps, total_ms, world, scale)

    # roofline of the dominant kernel: algorithmic work per launch / mean launch duration
    mean_ms = sum(times) / len(times)
    achieved = work / (mean_ms * 1e-3) / scale
    if w["kind"] in ("decode", "decode_paged"):
        bound, peak, punit = "hbm", peaks["hbm_gbs"], "GB/s"
    else:
        bound, peak, punit = "tensor", peaks["bf16_tflops"], "TFLOP/s"
        fp8_peak = None
        if w["kind"] == "fwd_fp8":
            fp8_peak = fp8_gemm_peak()
            # measured here; if the FP8 GEMM cannot run, the bf16 figure times the nominal
            # ratio 4.5 / 2.25
            peak = fp8_peak if fp8_peak else round(2.0 * peaks["bf16_tflops"], 1)
        if w["kind"] == "fwd_f32":
            # fp32 FMA on the CUDA cores: 148 SMs x 128 FMA lanes x 2 FLOP x 1965 MHz (the
            # maximum SM clock), no tensor core
            bound, peak = "alu", FP32_FMA_PEAK_TFLOPS
    tr = NCU_TRAFFIC.get(name)
    traffic = tr["bytes"] if tr and tr["src"] == kernel_sources_hash(family_of(w)) else None
    source = peak_kind + (" burst" if bound == "tensor" else "")
    if w["kind"] == "fwd_fp8":
        source = ("measured in this run: torch._scaled_mm E4M3 8192^3, best of 10" if fp8_peak
                  else peak_kind + " burst bf16 x 2 (nominal FP8 / BF16 ratio)")
    if bound == "alu":
        source = "derived: 148 SMs x 128 fp32 FMA/clk x 2 FLOP x 1965 MHz"
    roof = {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": punit,
            "frac": round(achieved / peak, 4) if peak else None, "traffic": traffic,
            "peak_source": source}
    if bound in NOMINAL and w["kind"] != "fwd_fp8":
        roof["peak_nominal"] = NOMINAL[bound]
        roof["frac_nominal"] = round(achieved / NOMINAL[bound], 4)

    # end to end through the public API with host buffers: H2D of inputs, call, D2H of results
    e2e = end_to_end(wl, work, scale, unit, max(3, min(steps, 20)), flush, world, dist_on)
    return dict(wl=wl, work=work, unit=unit, value=value, ms_per_step=ms_per_step,
                roofline=roof, e2e=e2e, clocks=sampler.report(),
                launches=wl.launches_per_step * steps, steps=steps)


def end_to_end(wl, work, scale, unit, steps, flush, world, dist_on):
    """The metric through the public API from pinned host buffers: every step copies its inputs
    host -> device, runs the call and copies its results device -> host.

    Pipelined: the copies run on their own streams, two device copies of
    the inputs alternate, so the upload of step i + 1 overlaps the call and the download of step
    i; a call waits for its inputs and for the download of the previous results (the outputs
    are single-buffered).  Serial: each step's upload, call and download one after the other on
    one stream.  The reported value is the faster of the two; both are kept in the record.  An
    L2 flush precedes every call."""
    import torch

    host_in = [t.cpu().pin_memory() for t in wl.inputs]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in wl.outputs]
    dev_in = [[torch.empty_like(t) for t in wl.inputs] for _ in range(2)]
    h2d_bytes = sum(t.numel() * t.element_size() for t in host_in)
    d2h_bytes = sum(t.numel() * t.element_size() for t in host_out)

    def serial_step():
        for dst, src in zip(dev_in[0], host_in):
            dst.copy_(src, non_blocking=True)
        wl.run(dev_in[0])
        for dst, src in zip(host_out, wl.outputs):
            dst.copy_(src, non_blocking=True)

    serial = timed_loop(serial_step, steps, 2, flush, dist_on)
    serial_ms = max_over_ranks(sum(serial), dist_on) / len(serial)

    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined(n):
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_up = [torch.cuda.Event() for _ in range(n)]
        ev_down = [torch.cuda.Event() for _ in range(n)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        up.wait_stream(comp)
        start.record(up)
        for i in range(n):
            buf = dev_in[i & 1]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_comp[i - 2])  # the call two steps back read this buffer
                for dst, src in zip(buf, host_in):
                    dst.copy_(src, non_blocking=True)
                ev_up[i].record(up)
            comp.wait_event(ev_up[i])
            if i >= 1:
                comp.wait_event(ev_down[i - 1])  # the previous results have left
            flush.zero_()
            wl.run(buf)
            ev_comp[i].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(ev_comp[i])
                for dst, src in zip(host_out, wl.outputs):
                    dst.copy_(src, non_blocking=True)
                ev_down[i].record(down)
        end.record(down)
        comp.wait_stream(down)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    pipelined(2)  # warm-up
    if dist_on:
        import torch.distributed as dist

        dist.barrier()
    total = max_over_ranks(pipelined(steps), dist_on)
    if dist_on:
        dist.barrier()
    ms = total / steps
    # the faster of the two schedules is the end-to-end figure (for a small problem the
    # pipelined loop's extra stream and event work on the host can cost more than it hides)
    best = min(ms, serial_ms)
    return {"value": round(world * work / (best * 1e-3) / scale, 3), "unit": unit,
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
            "ms_per_step": round(best, 4), "steps": steps,
            "schedule": "pipelined" if ms <= serial_ms else "serial",
            "pipelined": "upload of step i+1 overlaps the call and download of step i",
            "pipelined_ms_per_step": round(ms, 4),
            "pipelined_value": round(world * work / (ms * 1e-3) / scale, 3),
            "serial_ms_per_step": round(serial_ms, 4),
            "serial_value": round(world * work / (serial_ms * 1e-3) / scale, 3)}


# ----------------------------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------------------------
def oracle_sample(name, budget_s, seed=0, host=None):
    """Time the fp64 oracle on a random sample of the workload's output rows (prefill) or
    sequences (decode), growing the sample until it has run for about ``budget_s`` seconds.
    Returns (work units done, seconds, cores, description)."""
    import numpy as np

    import synth
    from exact_io_aware_82_b200 import accounting as acc
    from oracle import oracle as O

    w = WORKLOADS[name]
    rng = np.random.default_rng(seed)
    cores = O.num_threads()
    d = w["d"]
    scale = 1 / math.sqrt(d)
    B, Hq, Hkv, N = w["B"], w["Hq"], w["Hkv"], w["N"]
    G = Hq // Hkv

    def draw(tid, shape):
        if w["kind"] == "fwd_f32":
            return synth.normal_f32(w["seed"], tid, shape).astype(np.float64)
        if w["kind"] == "fwd_fp8":
            codes, sc = synth.normal_e4m3(w["seed"], tid, shape)
            return synth.e4m3_bits_to_f32(codes).astype(np.float64) * sc.astype(np.float64)[..., None, None]
        return synth.bf16_bits_to_f32(synth.normal_bf16_bits(w["seed"], tid, shape)).astype(np.float64)

    if w["kind"] == "fwd_varlen":
        # one sequence at a time, random rows of it
        done, secs, rows_done = 0, 0.0, 0
        lens = w["lens"]
        while secs < budget_s and rows_done < sum(lens):
            si = int(rng.integers(0, len(lens)))
            n = lens[si]
            base = sum(lens[:si])
            q = _draw_rows(w, synth.Q_ID, base, n, Hq, d)
            k = _draw_rows(w, synth.K_ID, base, n, Hkv, d)
            v = _draw_rows(w, synth.V_ID, base, n, Hkv, d)
            rows = rng.integers(0, Hq * n, size=min(64, Hq * n))
            t0 = time.perf_counter()
            O.attention_rows(q, k, v, rows, w["mask"], w["window"], w["n_sink"], scale)
            secs += time.perf_counter() - t0
            done += sum(4 * d * acc.visible_pairs(1, int(r % n) + 1, w["mask"], w["window"], w["n_sink"])
                        for r in rows)
            rows_done += len(rows)
        return done, secs, cores, "%d output rows drawn at random from random sequences of the batch" % rows_done
    if w["kind"] == "decode":
        # one sequence at a time: its query (Hq x d) against its own Hkv heads of the cache
        done, secs, seqs = 0, 0.0, 0
        qall = draw(synth.Q_ID, (B, Hq, 1, d))
        while secs < budget_s and seqs < B:
            b = int(rng.integers(0, B))
            # draw only this sequence's cache slice: element indices of [b][:][:][:]
            kk = _draw_slice(w, synth.K_ID, b, Hkv * N * d).reshape(1, Hkv, N, d)
            vv = _draw_slice(w, synth.V_ID, b, Hkv * N * d).reshape(1, Hkv, N, d)
            t0 = time.perf_counter()
            O.attention(qall[b:b + 1], kk, vv, FULL, scale=scale)
            secs += time.perf_counter() - t0
            done += acc.decode_bytes(1, Hq, Hkv, N, d)
            seqs += 1
        return done, secs, cores, "%d of %d sequences (all %d heads, %d cached keys each)" % (
            seqs, B, Hq, N)

    if w["kind"] == "bwd":
        # one (b, kv head) slice at a time: the gradients of a slice depend on that slice only
        done, secs, slices = 0, 0.0, 0
        while secs < budget_s and slices < B * Hkv:
            b, hk = int(rng.integers(0, B)), int(rng.integers(0, Hkv))
            qs = np.stack([_draw_slice(w, synth.Q_ID, b * Hq + hk * G + g, N * d) for g in range(G)])
            ds = np.stack([_draw_slice(w, synth.DO_ID, b * Hq + hk * G + g, N * d) for g in range(G)])
            kk = _draw_slice(w, synth.K_ID, b * Hkv + hk, N * d).reshape(1, 1, N, d)
            vv = _draw_slice(w, synth.V_ID, b * Hkv + hk, N * d).reshape(1, 1, N, d)
            t0 = time.perf_counter()
            O.attention_bwd(qs.reshape(1, G, N, d), kk, vv, ds.reshape(1, G, N, d), w["mask"],
                            w["window"], w["n_sink"], scale)
            secs += time.perf_counter() - t0
            done += acc.attn_bwd_flops(1, G, N, N, d, w["mask"], w["window"], w["n_sink"])
            slices += 1
        return done, secs, cores, "%d of %d (b, kv head) slices (%d query heads, %d rows each)" % (
            slices, B * Hkv, G, N)
    if w["kind"] == "decode_paged":
        # one sequence at a time, its keys gathered from its pages in block-table order
        ps = w["page_size"]
        table = paged_table(w)
        page_elems = ps * Hkv * d
        done, secs, seqs = 0, 0.0, 0
        qall = draw(synth.Q_ID, (B, Hq, 1, d))
        while secs < budget_s and seqs < B:
            b = int(rng.integers(0, B))
            kk = np.concatenate([_draw_slice(w, synth.K_ID, int(p), page_elems).reshape(ps, Hkv, d)
                                 for p in table[b]])
            vv = np.concatenate([_draw_slice(w, synth.V_ID, int(p), page_elems).reshape(ps, Hkv, d)
                                 for p in table[b]])
            kk = kk[:N].transpose(1, 0, 2)[None]
            vv = vv[:N].transpose(1, 0, 2)[None]
            t0 = time.perf_counter()
            O.attention(qall[b:b + 1], kk, vv, FULL, scale=scale)
            secs += time.perf_counter() - t0
            done += acc.decode_paged_bytes(1, Hq, Hkv, N, d, ps)
            seqs += 1
        return done, secs, cores, "%d of %d sequences (all %d heads, %d cached keys in %d-key pages)" % (
            seqs, B, Hq, N, ps)

    if w["kind"] in ("fwd", "fwd_block_sparse"):
        # one (b, query head) slice at a time (its Q slice and its kv head's K, V slices are
        # drawn alone, not timed), a growing batch of its rows
        bm = None
        if w["kind"] == "fwd_block_sparse":
            assert w["mask"] == FULL, "the block-sparse sample cuts query blocks of a full mask"
            nt = -(-N // 128)
            bm = synth.block_layout_bigbird(w["seed"], nt, nt, w["n_random"])
        done_rows, secs, work, batch = 0, 0.0, 0, 64
        while secs < budget_s and done_rows < B * Hq * N:
            b, h = int(rng.integers(0, B)), int(rng.integers(0, Hq))
            qq = _draw_slice(w, synth.Q_ID, b * Hq + h, N * d).reshape(1, 1, N, d)
            kk = _draw_slice(w, synth.K_ID, b * Hkv + h // G, N * d).reshape(1, 1, N, d)
            vv = _draw_slice(w, synth.V_ID, b * Hkv + h // G, N * d).reshape(1, 1, N, d)
            if bm is None:
                rows = rng.integers(0, N, size=batch)
                t0 = time.perf_counter()
                O.attention_rows(qq, kk, vv, rows, w["mask"], w["window"], w["n_sink"], scale)
                secs += time.perf_counter() - t0
                work += sum(4 * d * acc.visible_pairs(1, int(r) + 1, w["mask"], w["window"],
                                                      w["n_sink"]) if w["mask"] != FULL
                            else 4 * d * N for r in rows)
                done_rows += batch
            else:
                # whole 128-row query blocks: the layout row of block qt applies to all of them
                for qt in rng.integers(0, bm.shape[1], size=max(1, batch // 128)):
                    lo, hi = int(qt) * 128, min(N, int(qt) * 128 + 128)
                    t0 = time.perf_counter()
                    O.attention_block_sparse(qq[:, :, lo:hi], kk, vv, bm[:, qt:qt + 1], FULL,
                                             scale=scale)
                    secs += time.perf_counter() - t0
                    keys = sum(min(128, N - 128 * j) for j in range(bm.shape[2]) if bm[0, qt, j])
                    work += 4 * d * (hi - lo) * keys
                    done_rows += hi - lo
            batch = min(batch * 2, 4096)
        return work, secs, cores, "%d output rows of random (b, head) slices, drawn at random " \
            "(with replacement)%s" % (done_rows, " in whole 128-row blocks" if bm is not None
                                      else "")

    q = draw(synth.Q_ID, (B, Hq, N, d)) if host is None else host[0]
    k = draw(synth.K_ID, (B, Hkv, N, d)) if host is None else host[1]
    v = draw(synth.V_ID, (B, Hkv, N, d)) if host is None else host[2]
    total_rows = B * Hq * N
    done_rows, secs, work = 0, 0.0, 0
    batch = 64
    while secs < budget_s and done_rows < total_rows:
        rows = rng.integers(0, total_rows, size=batch)
        t0 = time.perf_counter()
        O.attention_rows(q, k, v, rows, w["mask"], w["window"], w["n_sink"], scale)
        secs += time.perf_counter() - t0
        i = rows % N
        for r in i:
            work += 4 * d * acc.visible_pairs(1, int(r) + 1, w["mask"], w["window"], w["n_sink"]) \
                if w["mask"] != FULL else 4 * d * N
        done_rows += batch
        batch = min(batch * 2, 4096)
    return work, secs, cores, "%d output rows drawn at random (with replacement) from the %d rows" % (
        done_rows, total_rows)


def _draw_rows(w, tid, base, n, H, d):
    """Rows [base, base + n) of a packed [total][H][d] tensor as a [1][H][n][d] fp64 array."""
    import numpy as np

    import synth

    count = n * H * d
    x = synth._box_muller(synth.splitmix64_np(synth._keys(w["seed"], tid, base * H * d, count)))
    bits = synth.f32_to_bf16_bits(x.astype(np.float32))
    return synth.bf16_bits_to_f32(bits).astype(np.float64).reshape(n, H, d).transpose(1, 0, 2)[None]


def _draw_slice(w, tid, b, count):
    """Elements [b * count, (b + 1) * count) of a tensor (one sequence's cache), as fp64."""
    import numpy as np

    import synth

    x = synth._box_muller(synth.splitmix64_np(synth._keys(w["seed"], tid, b * count, count)))
    bits = synth.f32_to_bf16_bits(x.astype(np.float32))
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def cpu_baseline(name, budget_s=12.0):
    work, secs, cores, desc = oracle_sample(name, budget_s)
    _, unit, scale = work_of(WORKLOADS[name])
    return {"value": round(work / secs / scale, 6), "unit": unit, "cores": cores,
            "kind": "oracle", "sample": desc + ", %.1f s" % secs}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    name = HEADLINE if args.workload in (None, "all") else args.workload
    w = WORKLOADS[name]
    _, unit, scale = work_of(w)
    per_step = []
    for i in range(args.warmup + args.steps):
        work, secs, cores, desc = oracle_sample(name, 1.0, seed=i)
        if i >= args.warmup:
            per_step.append((work, secs))
    work = sum(x for x, _ in per_step)
    secs = sum(s for _, s in per_step)
    value = work / secs / scale
    line = {"metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000 * secs / len(per_step), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(name, w, 1), "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores,
                             "kind": "oracle",
                             "sample": "each step: random output rows or sequences of the "
                                       "workload for about 1 s of oracle time"},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, help="one of %s, or 'all'" % ", ".join(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 runs under torch.distributed.run with N processes")
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU fallback)")
    torch.cuda.set_device(local)
    dist_on = world > 1
    if dist_on:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from exact_io_aware_82_b200 import build

    if rank == 0:
        build.build()
    if dist_on:
        torch.distributed.barrier()
    peaks, peak_kind = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    names = ([n for n in WORKLOADS if n not in PROFILING_ONLY]
             if args.workload == "all" else [args.workload or HEADLINE])
    for name in names:
        r = measure_ours(name, args.steps, args.warmup, rank, world, dist_on, flush, peaks,
                         peak_kind)
        w = WORKLOADS[name]
        line = {"metric": METRIC, "value": round(r["value"], 3), "unit": r["unit"],
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(r["ms_per_step"], 5), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None,
                "dtype": {"fwd_f32": "f32", "fwd_fp8": "e4m3 (fp32 accumulate, bf16 out)"}.get(
                    w["kind"], "bf16"),
                "data": "synthetic (iid N(0,1), seeded counter-based generator)",
                "config": config_of(name, w, world), "roofline": r["roofline"], "e2e": r["e2e"],
                "gpu_launches": r["launches"], "clocks": r["clocks"]}
        del r["wl"]
        cpu_on = rank == 0 and world == 1 and not args.no_cpu_baseline
        if args.workload is None and name == HEADLINE:
            for key, xname, fixed in EXTRAS:
                x = measure_ours(xname, args.steps, args.warmup, rank, world, dist_on, flush,
                                 peaks, peak_kind, 0.0 if fixed else MIN_TIMED_MS)
                del x["wl"]
                sub = {"workload": xname, "config": config_of(xname, WORKLOADS[xname], world),
                       "value": round(x["value"], 3), "unit": x["unit"], "steps": x["steps"],
                       "ms_per_step": round(x["ms_per_step"], 5), "roofline": x["roofline"],
                       "e2e": x["e2e"], "clocks": x["clocks"], "gpu_launches": x["launches"]}
                if cpu_on:
                    sub["cpu_baseline"] = cpu_baseline(xname, budget_s=8.0)
                line[key] = sub
        if cpu_on:
            line["cpu_baseline"] = cpu_baseline(name)
        if rank == 0:
            print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
