"""Benchmark of the hybrid sliding-window attention hot path on B200.

Default workload (one JSON line): Mistral-shaped sliding-window prefill of one 16K-token
chunk, B=2, N=16384, W=4096, Hq=32, Hkv=8, head_dim=128, bf16 Q/K/V ~ N(0,1)/sqrt(2) from
the seeded generator. One step = swa_prefill_fwd (band attention on tensor cores) +
kv_pool_append (commit of the chunk's last W tokens into the rolling buffer). Useful
FLOPs count only the (query, key) pairs inside the band: 4 * d * pairs * Hq * B.

Secondary results in the same line (unless --no-secondary): the 512-token single-layer
cases (W = 128, 512, 1), the hybrid 16K chunk after a 131072-token prefix (one SWA layer
W=128 and one paged full layer), and the hybrid decode batch (256 sequences, log-uniform
context lengths in [1K, 256K], 4 query tokens each, 6 SWA layers + 1 full layer) with
window_safe_len over 4096 requests.

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no data-path
collective); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np
import torch

import synth

METRIC = "SWA/full prefill TFLOP/s (% BF16 peak); hybrid decode KV GB/s (% HBM peak)"
ATOL_MAX, ATOL_MEAN = 2e-2, 2e-3  # attention parity against the fp64 oracle (max-abs, mean-abs)


def parity_ok(max_err, mean_err) -> bool:
    return max_err is not None and max_err <= ATOL_MAX and mean_err <= ATOL_MEAN
SEED = 20261202


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
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
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Largest value over all ranks (the step time of a weak-scaling run is the slowest rank's)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, ws: int, ms_max: float, scale: float) -> float:
    """Whole-job throughput: every rank processes the same units; time is the slowest rank's."""
    return units_per_rank * ws / ms_max / scale


def sum_over_ranks(x: float, ws: int) -> float:
    """Units of work of all ranks together (each rank counts its own)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------ workloads

def fp8_values(oracle_mod, x, scales):
    """The values an FP8 pool holds for bf16 rows x [n, Hkv, d] stored with one scale per KV head:
    the oracle's decode of every code (as a 256-entry table) times the head's scale, which is
    oracle.e4m3_dequantize(oracle.e4m3_quantize(.)) at table-lookup speed."""
    lut = oracle_mod.e4m3_decode(np.arange(256, dtype=np.uint8))
    out = np.empty(tuple(x.shape), dtype=np.float64)
    for g in range(x.shape[1]):
        sc = np.float32(scales[g])
        out[:, g] = lut[oracle_mod.e4m3_quantize(x[:, g].contiguous(), float(sc))] * np.float64(sc)
    return out


def gen(tag, layer, seq, pos0, n, h, d, sigma, device):
    return synth.normal_bf16_rows(SEED, synth.stream_id(tag, layer, seq), pos0, n, h * d, sigma, device).view(n, h, d)


class SwaPrefill16k:
    """Mistral-shaped SWA prefill of one 16K chunk (B=2, N=16384, W=4096, Hq=32, Hkv=8, d=128)."""
    name = "swa_prefill_16k_B2_W4096_Hq32_Hkv8_d128"

    @staticmethod
    def config(ws, B=2, N=16384, W=4096, Hq=32, Hkv=8, d=128, shard="replicas", gather_o=False):
        """The config dict of this workload's JSON line (the same for both arms)."""
        if shard == "heads":
            par = (f"KV heads split over {ws} ranks ({Hkv // ws} KV / {Hq // ws} query heads each)" +
                   (", O all-gathered (NCCL) every step" if gather_o else ", O left head-sharded"))
        else:
            par = f"independent batches x{ws}"
        return {"workload": SwaPrefill16k.name, "B_per_gpu": B, "seq_len": N, "window": W, "Hq": Hq,
                "Hkv": Hkv, "head_dim": d, "parallelism": par,
                "step": "swa_prefill_fwd + kv_pool_append(ring commit)",
                "l2": "inputs larger than L2 (Q 268 MB + K/V 134 MB + O 268 MB per step)"}

    def __init__(self, hs, B=2, N=16384, W=4096, Hq=32, Hkv=8, d=128, seq_offset=0, heads=None, gather_o=False):
        """heads = (g0, g1): this rank's KV heads when the problem is split by KV head (its query
        heads are [g0 G, g1 G)); the data of a head are those of the unsplit problem."""
        self.hs = hs
        self.B, self.N, self.W, self.Hq, self.Hkv, self.d = B, N, W, Hq, Hkv, d
        self.sigma = 2 ** -0.5
        self.seq_offset = seq_offset
        G = Hq // Hkv
        self.g0, self.g1 = heads if heads is not None else (0, Hkv)
        self.hkv_l, self.hq_l = self.g1 - self.g0, (self.g1 - self.g0) * G
        h0, h1 = self.g0 * G, self.g1 * G
        dev = "cuda"
        self.q = torch.stack([gen(synth.TAG_Q, 0, seq_offset + b, 0, N, Hq, d, self.sigma, dev)[:, h0:h1]
                              for b in range(B)]).contiguous()
        self.k = torch.stack([gen(synth.TAG_K, 0, seq_offset + b, 0, N, Hkv, d, self.sigma, dev)[:, self.g0:self.g1]
                              for b in range(B)]).contiguous()
        self.v = torch.stack([gen(synth.TAG_V, 0, seq_offset + b, 0, N, Hkv, d, self.sigma, dev)[:, self.g0:self.g1]
                              for b in range(B)]).contiguous()
        self.o = torch.empty_like(self.q)
        self.pool = hs.kv_pool_create(hs.PoolDesc(1, 0, W, self.hkv_l, d, B, 0))
        self.start = torch.zeros(B, dtype=torch.int64, device=dev)
        self.seq_ids = torch.arange(B, dtype=torch.int32, device=dev)
        pairs = W * (W + 1) // 2 + (N - W) * W if N >= W else N * (N + 1) // 2
        self.flops = 4 * d * pairs * self.hq_l * B  # this rank's share (the whole problem unless split)
        self.tail = min(N, W)
        self.gather_o = gather_o and torch.distributed.is_initialized()
        if self.gather_o:
            ws = torch.distributed.get_world_size()
            self.o_all = torch.empty((ws,) + tuple(self.o.shape), dtype=self.o.dtype, device=dev)

    def step(self, ev=None):
        hs = self.hs
        if ev is not None:
            ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
            ev[-1][0].record()
        hs.swa_prefill_fwd(self.pool, 0, self.q, self.k, self.v, o=self.o)
        if ev is not None:
            ev[-1][1].record()
        # commit the chunk into the rolling buffer (only its last W tokens land)
        hs.kv_pool_append(self.pool, 0, self.k, self.v, self.start, seq_ids=self.seq_ids)
        if self.gather_o:
            # every rank gets every head's output: rank-major slices [rank][B][N][Hq / ranks][d]
            torch.distributed.all_gather_into_tensor(self.o_all, self.o)

    launches_per_step = 2

    def e2e_setup(self):
        self.hq = self.q.cpu().pin_memory()
        self.hk = self.k.cpu().pin_memory()
        self.hv = self.v.cpu().pin_memory()
        self.ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = (self.hq.numel() + self.hk.numel() + self.hv.numel()) * 2
        self.d2h = self.ho.numel() * 2
        # Serving-loop form: two device buffer sets, uploads on one copy stream and downloads on
        # another, so step i+1's inputs and step i-1's output cross PCIe (both directions at once)
        # while step i computes. Every step still uploads its own inputs and downloads its own O.
        self.pipelined = not self.gather_o
        if self.pipelined:
            self.bufs = [(self.q, self.k, self.v, self.o),
                         tuple(torch.empty_like(t) for t in (self.q, self.k, self.v, self.o))]
            self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
            self.done_reading = [None, None]  # compute of the last step that read buffer set b
            self.done_out = [None, None]      # download of the last step that wrote O of set b
            self.n_e2e = 0

    def e2e_begin(self):
        if self.pipelined:
            cur = torch.cuda.current_stream()
            self.s_in.wait_stream(cur)
            self.s_out.wait_stream(cur)

    def e2e_step(self):
        if not self.pipelined:
            self.q.copy_(self.hq, non_blocking=True)
            self.k.copy_(self.hk, non_blocking=True)
            self.v.copy_(self.hv, non_blocking=True)
            self.step()
            self.ho.copy_(self.o, non_blocking=True)
            return
        b = self.n_e2e % 2
        self.n_e2e += 1
        q, k, v, o = self.bufs[b]
        cur = torch.cuda.current_stream()
        with torch.cuda.stream(self.s_in):
            if self.done_reading[b] is not None:
                self.s_in.wait_event(self.done_reading[b])
            q.copy_(self.hq, non_blocking=True)
            k.copy_(self.hk, non_blocking=True)
            v.copy_(self.hv, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(self.s_in)
        cur.wait_event(ready)
        if self.done_out[b] is not None:
            cur.wait_event(self.done_out[b])
        self.hs.swa_prefill_fwd(self.pool, 0, q, k, v, o=o)
        self.hs.kv_pool_append(self.pool, 0, k, v, self.start, seq_ids=self.seq_ids)
        comp = torch.cuda.Event()
        comp.record(cur)
        self.done_reading[b] = comp
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(comp)
            self.ho.copy_(o, non_blocking=True)
            out = torch.cuda.Event()
            out.record(self.s_out)
            self.done_out[b] = out

    def e2e_end(self):
        if self.pipelined:
            cur = torch.cuda.current_stream()
            cur.wait_stream(self.s_in)
            cur.wait_stream(self.s_out)

    def check_sample(self, oracle, rows=(0, 1, 127, 128, 4095, 4096, 9999, 16383)):
        """Sampled rows (all heads, both sequences) against the oracle; returns (max, mean) abs error."""
        errs = []
        for b in range(self.B):
            lo = max(0, min(rows) - self.W + 1)
            hi = max(rows) + 1
            k = gen(synth.TAG_K, 0, self.seq_offset + b, lo, hi - lo, self.Hkv, self.d, self.sigma, "cpu")
            v = gen(synth.TAG_V, 0, self.seq_offset + b, lo, hi - lo, self.Hkv, self.d, self.sigma, "cpu")
            qr = torch.stack([gen(synth.TAG_Q, 0, self.seq_offset + b, r, 1, self.Hq, self.d, self.sigma, "cpu")[0]
                              for r in rows])
            ref = oracle.attention(qr, np.array(rows), k, v, self.W, key_base=lo)
            G = self.Hq // self.Hkv
            ref = ref[:, self.g0 * G:self.g1 * G]  # this rank's heads
            got = self.o[b, list(rows)].float().cpu().double().numpy()
            errs.append(np.abs(got - ref))
        e = np.concatenate([x.ravel() for x in errs])
        return float(e.max()), float(e.mean())

    def oracle_sample(self, oracle, budget_s=10.0, block=32, threads=None):
        """Time the oracle on blocks of query rows (all heads, full W-key windows) taken from the end of
        sequence 0 until about budget_s seconds have passed; returns (seconds, flops, rows)."""
        max_rows = 2048
        rows_all = np.arange(self.N - max_rows, self.N)
        lo = rows_all[0] - self.W + 1
        k = gen(synth.TAG_K, 0, self.seq_offset, lo, self.N - lo, self.Hkv, self.d, self.sigma, "cpu")
        v = gen(synth.TAG_V, 0, self.seq_offset, lo, self.N - lo, self.Hkv, self.d, self.sigma, "cpu")
        q = gen(synth.TAG_Q, 0, self.seq_offset, rows_all[0], max_rows, self.Hq, self.d, self.sigma, "cpu")
        done, dt = 0, 0.0
        while dt < budget_s and done < max_rows:
            r = rows_all[done:done + block]
            t0 = time.perf_counter()
            oracle.attention(q[done:done + block], r, k, v, self.W, key_base=lo, n_threads=threads)
            dt += time.perf_counter() - t0
            done += len(r)
        flops = 4 * self.d * done * self.W * self.Hq
        return dt, flops, done


class LongContext1M:
    """Final 16K chunk of a 1,048,576-token prefill through the 70-layer hybrid schedule: 60 SWA
    layers (W=128, prefix from the rolling buffer) and 10 full layers (paged pools holding all
    1,048,576 tokens each), B=1, Hq=64, Hkv=8, d=128, bf16 N(0,1). One step = the 70 attention
    calls of the chunk (the K/V of the chunk are committed to the full pools at set-up; the rings
    keep the pre-chunk state so every step sees the same prefix)."""
    name = "long_context_1m_final16k_60swaW128_10full_Hq64_Hkv8_d128"
    launches_per_step = 70

    def __init__(self, hs, seq_offset=0, N=1 << 20, Nc=16384, W=128, Hq=64, Hkv=8, d=128, n_swa=60, n_full=10):
        self.hs = hs
        self.N, self.Nc, self.W, self.Hq, self.Hkv, self.d = N, Nc, W, Hq, Hkv, d
        self.P = N - Nc
        self.n_swa, self.n_full = n_swa, n_full
        self.B = 1
        self.seq = 300 + seq_offset
        dev = "cuda"
        pages = N // 64
        self.pool = hs.kv_pool_create(hs.PoolDesc(n_swa, n_full, W, Hkv, d, 1, pages))
        perm = synth.permutation(SEED, synth.stream_id(synth.TAG_MISC, 6), pages).to(torch.int32)
        self.pt = perm.view(1, pages).to(dev)
        self.sid = torch.zeros(1, dtype=torch.int32, device=dev)
        self.start = torch.tensor([self.P], dtype=torch.int64, device=dev)
        self.q, self.k, self.v = {}, {}, {}
        for layer in range(n_swa):
            kp = gen(synth.TAG_K, layer, self.seq, self.P - W, W, Hkv, d, 1.0, dev)[None]
            vp = gen(synth.TAG_V, layer, self.seq, self.P - W, W, Hkv, d, 1.0, dev)[None]
            hs.kv_pool_append(self.pool, layer, kp, vp, torch.tensor([self.P - W], device=dev), seq_ids=self.sid)
            self.k[layer] = gen(synth.TAG_K, layer, self.seq, self.P, Nc, Hkv, d, 1.0, dev)[None]
            self.v[layer] = gen(synth.TAG_V, layer, self.seq, self.P, Nc, Hkv, d, 1.0, dev)[None]
        for f in range(n_full):
            layer = n_swa + f
            for c0 in range(0, N, 65536):
                m = min(65536, N - c0)
                kf = gen(synth.TAG_K, layer, self.seq, c0, m, Hkv, d, 1.0, dev)[None]
                vf = gen(synth.TAG_V, layer, self.seq, c0, m, Hkv, d, 1.0, dev)[None]
                hs.kv_pool_append(self.pool, layer, kf, vf, torch.tensor([c0], device=dev), page_table=self.pt)
        for layer in range(n_swa + n_full):
            self.q[layer] = gen(synth.TAG_Q, layer, self.seq, self.P, Nc, Hq, d, 1.0, dev)[None]
        self.o = torch.empty_like(self.q[0])
        torch.cuda.synchronize()
        # the pages give only the layer counts; run them interleaved 6 SWA : 1 full
        self.order = []
        for blk in range(n_full):
            self.order += [blk * (n_swa // n_full) + i for i in range(n_swa // n_full)] + [n_swa + blk]
        swa_pairs = Nc * W
        full_pairs = Nc * self.P + Nc * (Nc + 1) // 2
        self.flops_swa = 4 * d * swa_pairs * Hq * n_swa
        self.flops_full = 4 * d * full_pairs * Hq * n_full
        self.flops = self.flops_swa + self.flops_full
        self.full_flops_per_launch = 4 * d * full_pairs * Hq

    def step(self, ev=None):
        hs = self.hs
        for layer in self.order:
            if layer < self.n_swa:
                hs.swa_prefill_fwd(self.pool, layer, self.q[layer], self.k[layer], self.v[layer], o=self.o,
                                   start_pos=self.start, seq_ids=self.sid)
            else:
                if ev is not None:
                    ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                    ev[-1][0].record()
                hs.full_prefill_fwd(self.pool, layer, self.q[layer], self.pt, o=self.o, start_pos=self.start)
                if ev is not None:
                    ev[-1][1].record()

    def footprint(self):
        _, swa, full = self.hs.kv_pool_layout(self.pool.desc)
        slot = 2 * self.Hkv * self.d * 2
        return {"swa_bytes": swa, "full_bytes": full, "slots": (swa + full) // slot,
                "expected_slots_60W_plus_10N": self.n_swa * self.W + self.n_full * self.N}

    def check_sample(self, oracle):
        """Rows 0 and Nc-1 of the last full layer and rows of one SWA layer against the oracle."""
        errs = []
        layer = self.n_swa + self.n_full - 1
        self.hs.full_prefill_fwd(self.pool, layer, self.q[layer], self.pt, o=self.o, start_pos=self.start)
        rows = [0, self.Nc - 1]
        got = self.o[0, rows].float().cpu().double().numpy()
        k = gen(synth.TAG_K, layer, self.seq, 0, self.N, self.Hkv, self.d, 1.0, "cpu")
        v = gen(synth.TAG_V, layer, self.seq, 0, self.N, self.Hkv, self.d, 1.0, "cpu")
        q = gen(synth.TAG_Q, layer, self.seq, self.P, self.Nc, self.Hq, self.d, 1.0, "cpu")[rows]
        errs.append(np.abs(got - oracle.attention(q, self.P + np.array(rows), k, v, 0)).ravel())
        del k, v
        layer = 7
        self.hs.swa_prefill_fwd(self.pool, layer, self.q[layer], self.k[layer], self.v[layer], o=self.o,
                                start_pos=self.start, seq_ids=self.sid)
        rows = [0, 1, 127, 128, 9999, self.Nc - 1]
        got = self.o[0, rows].float().cpu().double().numpy()
        base = self.P - self.W + 1
        k = gen(synth.TAG_K, layer, self.seq, base, self.N - base, self.Hkv, self.d, 1.0, "cpu")
        v = gen(synth.TAG_V, layer, self.seq, base, self.N - base, self.Hkv, self.d, 1.0, "cpu")
        q = gen(synth.TAG_Q, layer, self.seq, self.P, self.Nc, self.Hq, self.d, 1.0, "cpu")[rows]
        errs.append(np.abs(got - oracle.attention(q, self.P + np.array(rows), k, v, self.W, key_base=base)).ravel())
        e = np.concatenate(errs)
        return float(e.max()), float(e.mean())

    def oracle_sample(self, oracle, budget_s=10.0, threads=None):
        """Time the oracle on rows of one SWA layer (full 128-key windows) until about budget_s."""
        layer, rows_max = 3, 4096
        base = self.P - self.W + 1
        k = gen(synth.TAG_K, layer, self.seq, base, self.N - base, self.Hkv, self.d, 1.0, "cpu")
        v = gen(synth.TAG_V, layer, self.seq, base, self.N - base, self.Hkv, self.d, 1.0, "cpu")
        q = gen(synth.TAG_Q, layer, self.seq, self.P, rows_max, self.Hq, self.d, 1.0, "cpu")
        done, dt = 0, 0.0
        while dt < budget_s and done < rows_max:
            r = np.arange(done, min(done + 256, rows_max))
            t0 = time.perf_counter()
            oracle.attention(q[r], self.P + r, k, v, self.W, key_base=base, n_threads=threads)
            dt += time.perf_counter() - t0
            done = int(r[-1]) + 1
        return dt, 4 * self.d * done * self.W * self.Hq, done


class HybridChunk131k:
    """One 16K-token chunk after a 131072-token cached prefix (B=1, Hq=64, Hkv=8, d=128, bf16 N(0,1)):
    kind 'swa' is the sliding-window layer (W=128; the 127 prefix keys it needs come from the
    rolling buffer) -- bandwidth-bound, its metric is bytes moved; kind 'full' is the full layer
    over all 147456 keys through a randomly permuted 64-token page table (the chunk appended
    first) -- tensor-bound, its metric is useful FLOPs."""
    launches_per_step = 1

    def __init__(self, hs, kind="swa", seq_offset=0, P=131072, Nc=16384, W=128, Hq=64, Hkv=8, d=128, fp8=False):
        self.hs, self.kind, self.fp8 = hs, kind, fp8
        self.P, self.Nc, self.W, self.Hq, self.Hkv, self.d = P, Nc, W, Hq, Hkv, d
        self.N, self.B = Nc, 1
        self.seq = 100 + seq_offset
        self.name = ("swa_chunk16k_after_131072_W128_Hq64_Hkv8_d128" if kind == "swa" else
                     "full_chunk16k_after_131072_paged_Hq64_Hkv8_d128") + ("_fp8kv" if fp8 else "")
        dev = "cuda"
        total = P + Nc
        pages = total // 64
        fmt = hs.HSWA_KV_FP8_E4M3 if fp8 else hs.HSWA_KV_BF16
        self.pool = hs.kv_pool_create(hs.PoolDesc(1, 1, W, Hkv, d, 1, pages, kv_format=fmt))
        if fp8:
            # per-head scales of amax / 448 for |x| <= 6, as in the decode batch
            u = synth.uniform_float64(SEED, synth.stream_id(synth.TAG_MISC, 8, seq_offset), 4 * Hkv)
            self.scales = (6.0 / 448.0 * (0.75 + 0.5 * u)).to(torch.float32).view(2, 2, Hkv).numpy()
            for layer in range(2):
                self.pool.set_scales(layer, self.scales[layer, 0], self.scales[layer, 1])
        self.sid = torch.zeros(1, dtype=torch.int32, device=dev)
        self.start = torch.tensor([P], dtype=torch.int64, device=dev)
        if kind == "swa":
            kp = gen(synth.TAG_K, 0, self.seq, P - W, W, Hkv, d, 1.0, dev)[None]
            vp = gen(synth.TAG_V, 0, self.seq, P - W, W, Hkv, d, 1.0, dev)[None]
            hs.kv_pool_append(self.pool, 0, kp, vp, torch.tensor([P - W], device=dev), seq_ids=self.sid)
            self.k = gen(synth.TAG_K, 0, self.seq, P, Nc, Hkv, d, 1.0, dev)[None]
            self.v = gen(synth.TAG_V, 0, self.seq, P, Nc, Hkv, d, 1.0, dev)[None]
            self.q = gen(synth.TAG_Q, 0, self.seq, P, Nc, Hq, d, 1.0, dev)[None]
            e = 1 if fp8 else 2  # bytes per ring element
            self.flops = (2 * Nc * Hq * d + 2 * Nc * Hkv * d) * 2 + 2 * (W - 1) * Hkv * d * e  # bytes (metric)
            self.useful_flops = 4 * d * Nc * W * Hq
        else:
            perm = synth.permutation(SEED, synth.stream_id(synth.TAG_MISC, 3), pages).to(torch.int32)
            self.pt = perm.view(1, pages).to(dev)
            for c0 in range(0, total, 16384):
                n = min(16384, total - c0)
                kf = gen(synth.TAG_K, 1, self.seq, c0, n, Hkv, d, 1.0, dev)[None]
                vf = gen(synth.TAG_V, 1, self.seq, c0, n, Hkv, d, 1.0, dev)[None]
                hs.kv_pool_append(self.pool, 1, kf, vf, torch.tensor([c0], device=dev), page_table=self.pt)
            self.q = gen(synth.TAG_Q, 1, self.seq, P, Nc, Hq, d, 1.0, dev)[None]
            self.flops = 4 * d * (Nc * P + Nc * (Nc + 1) // 2) * Hq
        self.o = torch.empty_like(self.q)
        torch.cuda.synchronize()

    def step(self, ev=None):
        hs = self.hs
        if ev is not None:
            ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
            ev[-1][0].record()
        if self.kind == "swa":
            hs.swa_prefill_fwd(self.pool, 0, self.q, self.k, self.v, o=self.o, start_pos=self.start, seq_ids=self.sid)
        else:
            hs.full_prefill_fwd(self.pool, 1, self.q, self.pt, o=self.o, start_pos=self.start)
        if ev is not None:
            ev[-1][1].record()

    def e2e_setup(self):
        self.h_in = [t.cpu().pin_memory() for t in ([self.q, self.k, self.v] if self.kind == "swa" else [self.q])]
        self.ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = sum(t.numel() * 2 for t in self.h_in)
        self.d2h = self.ho.numel() * 2

    def e2e_step(self):
        dev_in = [self.q, self.k, self.v] if self.kind == "swa" else [self.q]
        for h, d_ in zip(self.h_in, dev_in):
            d_.copy_(h, non_blocking=True)
        self.step()
        self.ho.copy_(self.o, non_blocking=True)

    def _ref_rows(self, rows):
        P, W, Hkv, d, Hq = self.P, self.W, self.Hkv, self.d, self.Hq
        if self.kind == "swa":
            base = P - W + 1
            k = gen(synth.TAG_K, 0, self.seq, base, self.Nc + W - 1, Hkv, d, 1.0, "cpu")
            v = gen(synth.TAG_V, 0, self.seq, base, self.Nc + W - 1, Hkv, d, 1.0, "cpu")
            q = gen(synth.TAG_Q, 0, self.seq, P, self.Nc, Hq, d, 1.0, "cpu")[rows]
            return q, k, v, W, base
        k = gen(synth.TAG_K, 1, self.seq, 0, P + self.Nc, Hkv, d, 1.0, "cpu")
        v = gen(synth.TAG_V, 1, self.seq, 0, P + self.Nc, Hkv, d, 1.0, "cpu")
        q = gen(synth.TAG_Q, 1, self.seq, P, self.Nc, Hq, d, 1.0, "cpu")[rows]
        return q, k, v, 0, 0

    def _deq(self, oracle, x, layer, kv):
        return fp8_values(oracle, x, self.scales[layer, kv])

    def check_sample(self, oracle):
        rows = [0, 1, 127, 128, 8191, self.Nc - 1] if self.kind == "swa" else [0, 5000, self.Nc - 1]
        self.step()
        q, k, v, w, base = self._ref_rows(rows)
        if self.fp8:
            # cached keys come from the FP8 pool; an SWA chunk's own keys are used as given
            layer = 0 if self.kind == "swa" else 1
            n_cached = self.W - 1 if self.kind == "swa" else k.shape[0]
            k64, v64 = k.double().numpy(), v.double().numpy()
            k64[:n_cached] = self._deq(oracle, k[:n_cached], layer, 0)
            v64[:n_cached] = self._deq(oracle, v[:n_cached], layer, 1)
            ref = oracle.attention_kv64(q, self.P + np.array(rows), k64, v64, w, key_base=base)
        else:
            ref = oracle.attention(q, self.P + np.array(rows), k, v, w, key_base=base)
        e = np.abs(self.o[0, rows].float().cpu().double().numpy() - ref)
        return float(e.max()), float(e.mean())

    def oracle_sample(self, oracle, budget_s=10.0, threads=None):
        """Time the oracle on blocks of rows of this layer until about budget_s; returns
        (seconds, units of the metric those rows account for, rows)."""
        rows_all = np.arange(self.Nc)
        q, k, v, w, base = self._ref_rows(rows_all)
        done, dt = 0, 0.0
        block = 512 if self.kind == "swa" else 2
        while dt < budget_s and done < self.Nc:
            r = rows_all[done:done + block]
            t0 = time.perf_counter()
            oracle.attention(q[r], self.P + r, k, v, w, key_base=base, n_threads=threads)
            dt += time.perf_counter() - t0
            done += len(r)
        if self.kind == "swa":
            units = self.flops * done / self.Nc
        else:
            units = 4 * self.d * self.Hq * sum(self.P + int(i) + 1 for i in rows_all[:done])
        return dt, units, done


class DecodeBatch:
    """Hybrid decode step: n sequences with context lengths log-uniform in [1K, 256K], 4 query
    tokens each (1 + 3 multi-token-prediction drafts), 6 SWA layers on a 128-slot ring and 1 full
    layer on 64-token pages (seeded random page permutation), Hq=64, Hkv=8, d=128, bf16 N(0,1).
    One step = the 7 hybrid_decode_fwd calls. The metric counts the bytes the step must read
    (K/V of every cached key in every window, plus Q, the new K/V and O)."""
    launches_per_step = 7 * 3  # plan + decode (+ merge on the full layer) per call

    @staticmethod
    def batch_lens(n=256, seq_offset=0):
        """Context lengths of the batch: log-uniform in [1K, 256K] from the seed."""
        u = synth.uniform_float64(SEED, synth.stream_id(synth.TAG_MISC, 4, seq_offset), n)
        return torch.floor(torch.exp(math.log(1024) + u * (math.log(262144) - math.log(1024)))).to(torch.int64)

    def __init__(self, hs, n=256, seq_offset=0, Hq=64, Hkv=8, d=128, W=128, nq=4, n_swa=6, fp8=False, select=None):
        """select: indices of the batch's sequences this rank holds when decode is split by sequence
        (None: all of them); a sequence's data are those of the unsplit batch."""
        self.hs = hs
        dev = "cuda"
        self.Hq, self.Hkv, self.d, self.W, self.nq, self.n_swa = Hq, Hkv, d, W, nq, n_swa
        self.fp8 = fp8
        self.name = f"hybrid_decode_{n}seq_L1K-256K_6swa_1full_Hq64_Hkv8_d128_4tok" + ("_fp8kv" if fp8 else "")
        all_lens = self.batch_lens(n, seq_offset)
        self.total_ctx = int(all_lens.sum())
        self.gidx = list(range(n)) if select is None else [int(i) for i in select]
        n = len(self.gidx)
        self.n = n
        self.base = 200 + seq_offset * 100000
        self.lens = all_lens[self.gidx]
        lens = self.lens
        self.S = int(lens.sum())
        pps = (lens + nq + 63) // 64
        total_pages = int(pps.sum())
        maxp = int(pps.max())
        fmt = hs.HSWA_KV_FP8_E4M3 if fp8 else hs.HSWA_KV_BF16
        self.pool = hs.kv_pool_create(hs.PoolDesc(n_swa, 1, W, Hkv, d, n, total_pages, kv_format=fmt))
        if fp8:
            # per-head scales of amax / 448 for |x| <= 6 (the N(0, 1) entries use the whole E4M3 range)
            u = synth.uniform_float64(SEED, synth.stream_id(synth.TAG_MISC, 7, seq_offset), 2 * (n_swa + 1) * Hkv)
            sc = (6.0 / 448.0 * (0.75 + 0.5 * u)).to(torch.float32).view(n_swa + 1, 2, Hkv).numpy()
            self.scales = sc
            for layer in range(n_swa + 1):
                self.pool.set_scales(layer, sc[layer, 0], sc[layer, 1])
        perm = synth.permutation(SEED, synth.stream_id(synth.TAG_MISC, 5, seq_offset), total_pages).to(torch.int32)
        pt = torch.zeros(n, maxp, dtype=torch.int32)
        off = 0
        for i in range(n):
            pt[i, :pps[i]] = perm[off:off + int(pps[i])]
            off += int(pps[i])
        self.pt = pt.to(dev)
        self.sid = torch.arange(n, dtype=torch.int32, device=dev)
        self.full_layer = n_swa
        for b in range(n):
            L = int(lens[b])
            sq = self.base + self.gidx[b]  # the sequence's data stream (its index in the whole batch)
            for c0 in range(0, L, 65536):
                m = min(65536, L - c0)
                k = gen(synth.TAG_K, self.full_layer, sq, c0, m, Hkv, d, 1.0, dev)[None]
                v = gen(synth.TAG_V, self.full_layer, sq, c0, m, Hkv, d, 1.0, dev)[None]
                hs.kv_pool_append(self.pool, self.full_layer, k, v, torch.tensor([c0], device=dev),
                                  page_table=self.pt[b:b + 1])
            for layer in range(n_swa):
                k = gen(synth.TAG_K, layer, sq, L - W, W, Hkv, d, 1.0, dev)[None]
                v = gen(synth.TAG_V, layer, sq, L - W, W, Hkv, d, 1.0, dev)[None]
                hs.kv_pool_append(self.pool, layer, k, v, torch.tensor([L - W], device=dev), seq_ids=self.sid[b:b + 1])
        self.ctx = lens.to(dev)
        self.maxL = int(lens.max())
        self.qs, self.kn, self.vn = [], [], []
        for layer in range(n_swa + 1):
            self.qs.append(torch.stack([gen(synth.TAG_Q, layer, self.base + self.gidx[b], int(lens[b]), nq, Hq, d,
                                            1.0, dev) for b in range(n)]))
            self.kn.append(torch.stack([gen(synth.TAG_K, layer, self.base + self.gidx[b], int(lens[b]), nq, Hkv, d,
                                            1.0, dev) for b in range(n)]))
            self.vn.append(torch.stack([gen(synth.TAG_V, layer, self.base + self.gidx[b], int(lens[b]), nq, Hkv, d,
                                            1.0, dev) for b in range(n)]))
        self.ws = torch.empty(hs.hybrid_decode_workspace_size(self.pool, n, nq, Hq, self.maxL), dtype=torch.uint8,
                              device=dev)
        self.outs = [torch.empty_like(self.qs[0]) for _ in range(n_swa + 1)]
        e = 1 if fp8 else 2  # bytes per cached K/V element
        self.kv_full = self.S * Hkv * d * e * 2
        self.kv_swa = n_swa * n * (W - 1) * Hkv * d * e * 2
        qo = n * nq * (Hq * 2 + Hkv * 2) * d * 2      # Q + O + new K + new V per layer
        self.bytes = self.kv_full + self.kv_swa + (n_swa + 1) * qo
        self.full_bytes_per_launch = self.kv_full + qo
        torch.cuda.synchronize()

    def step(self, ev=None):
        hs = self.hs
        for layer in range(self.n_swa):
            hs.hybrid_decode_fwd(self.pool, layer, self.qs[layer], self.kn[layer], self.vn[layer], self.ctx, self.maxL,
                                 self.ws, seq_ids=self.sid, o=self.outs[layer])
        if ev is not None:
            ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
            ev[-1][0].record()
        L = self.full_layer
        hs.hybrid_decode_fwd(self.pool, L, self.qs[L], self.kn[L], self.vn[L], self.ctx, self.maxL, self.ws,
                             page_table=self.pt, o=self.outs[L])
        if ev is not None:
            ev[-1][1].record()

    def e2e_setup(self):
        self.h_in = [(q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory())
                     for q, k, v in zip(self.qs, self.kn, self.vn)]
        self.h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in self.outs]
        self.h2d = sum((q.numel() + k.numel() + v.numel()) * 2 for q, k, v in self.h_in)
        self.d2h = sum(o.numel() * 2 for o in self.h_out)

    def e2e_step(self):
        for (hq, hk, hv), q, k, v in zip(self.h_in, self.qs, self.kn, self.vn):
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
        self.step()
        for ho, o in zip(self.h_out, self.outs):
            ho.copy_(o, non_blocking=True)

    def check_sample(self, oracle):
        """All rows of the two shortest sequences and of the longest one (the most splits to merge) on
        the full layer, and of two sequences on an SWA layer. FP8 pools: against the oracle on the
        dequantized entries (new tokens included: they enter as the cache will hold them)."""
        lens, nq, Hq, Hkv, d, W = self.lens, self.nq, self.Hq, self.Hkv, self.d, self.W
        order = torch.argsort(lens)
        errs = []

        def attend(layer, b, lo, hi, window, key_base, L):
            sq = self.base + self.gidx[b]
            k = gen(synth.TAG_K, layer, sq, lo, hi - lo, Hkv, d, 1.0, "cpu")
            v = gen(synth.TAG_V, layer, sq, lo, hi - lo, Hkv, d, 1.0, "cpu")
            q = gen(synth.TAG_Q, layer, sq, L, nq, Hq, d, 1.0, "cpu")
            if not self.fp8:
                return oracle.attention(q, L + np.arange(nq), k, v, window, key_base=key_base)
            kd = fp8_values(oracle, k, self.scales[layer, 0])
            vd = fp8_values(oracle, v, self.scales[layer, 1])
            return oracle.attention_kv64(q, L + np.arange(nq), kd, vd, window, key_base=key_base)

        for b in [int(order[0]), int(order[1]), int(order[-1])]:
            L = int(lens[b])
            ref = attend(self.full_layer, b, 0, L + nq, 0, 0, L)
            errs.append(np.abs(self.outs[self.full_layer][b].float().cpu().double().numpy() - ref).ravel())
        for b in sorted({int(order[-1]), min(7, self.n - 1)}):
            L = int(lens[b])
            ref = attend(2, b, L - W + 1, L + nq, W, L - W + 1, L)
            errs.append(np.abs(self.outs[2][b].float().cpu().double().numpy() - ref).ravel())
        e = np.concatenate(errs)
        return float(e.max()), float(e.mean())

    def oracle_sample(self, oracle, budget_s=10.0, threads=None):
        """Time the oracle on whole sequences of the full layer, shortest first, until about budget_s;
        returns (seconds, bytes of K/V those rows read, sequences)."""
        order = torch.argsort(self.lens)
        dt, byts, done = 0.0, 0, 0
        for b in order.tolist():
            if dt >= budget_s:
                break
            L = int(self.lens[b])
            sq = self.base + self.gidx[b]
            k = gen(synth.TAG_K, self.full_layer, sq, 0, L + self.nq, self.Hkv, self.d, 1.0, "cpu")
            v = gen(synth.TAG_V, self.full_layer, sq, 0, L + self.nq, self.Hkv, self.d, 1.0, "cpu")
            q = gen(synth.TAG_Q, self.full_layer, sq, L, self.nq, self.Hq, self.d, 1.0, "cpu")
            t0 = time.perf_counter()
            oracle.attention(q, L + np.arange(self.nq), k, v, 0, n_threads=threads)
            dt += time.perf_counter() - t0
            byts += (L + self.nq) * self.Hkv * self.d * 2 * 2
            done += 1
        return dt, byts, done


def long_context_result(hs, oracle_mod, bf16_sus):
    """Config 5: the 70-layer step on the final 16K chunk of a 1M-token prefill (3 warm-up steps,
    1 timed step of ~5.6 s), with its full layers against the sustained bf16 peak."""
    wl = LongContext1M(hs)
    for _ in range(3):
        wl.step()
    torch.cuda.synchronize()
    ev = []
    a, b = torch.cuda.Event(True), torch.cuda.Event(True)
    a.record()
    wl.step(ev)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    ms_full = statistics.mean(x.elapsed_time(y) for x, y in ev)
    assert hs.hswa_pool_check_error(wl.pool) == 0
    fp = wl.footprint()
    mx, mean = wl.check_sample(oracle_mod)
    full_tf = wl.full_flops_per_launch / ms_full / 1e9
    res = {"workload": wl.name, "metric": "prefill TFLOP/s", "unit": "TFLOP/s",
           "value": round(wl.flops / ms / 1e9, 1), "ms": round(ms, 1),
           "full_layer_ms": round(ms_full, 2), "full_layer_tflops": round(full_tf, 1),
           "full_layer_frac_of_sustained_peak": round(full_tf / bf16_sus, 3),
           "footprint_slots": fp["slots"], "expected_slots_60W_plus_10N": fp["expected_slots_60W_plus_10N"],
           "steps": 1, "warmup": 3, "max_abs_err": mx, "mean_abs_err": mean}
    del wl
    torch.cuda.empty_cache()
    return res


def secondary_results(hs, oracle_mod, hbm, bf16, bf16_sus=None):
    out = []
    dev = "cuda"

    def t(fn, reps, warm=3):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(True), torch.cuda.Event(True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    # config 1: B=1, N=512, Hq=4, Hkv=1, d=64, W in {128, 512, 1}
    for W in (128, 512, 1):
        pool = hs.kv_pool_create(hs.PoolDesc(1, 0, W, 1, 64, 1, 0))
        q = gen(synth.TAG_Q, 10, 0, 0, 512, 4, 64, 1.0, dev)[None]
        k = gen(synth.TAG_K, 10, 0, 0, 512, 1, 64, 1.0, dev)[None]
        v = gen(synth.TAG_V, 10, 0, 0, 512, 1, 64, 1.0, dev)[None]
        o = torch.empty_like(q)
        ms = t(lambda: hs.swa_prefill_fwd(pool, 0, q, k, v, o=o), 50)
        kk = gen(synth.TAG_K, 10, 0, 0, 512, 1, 64, 1.0, "cpu")
        vv = gen(synth.TAG_V, 10, 0, 0, 512, 1, 64, 1.0, "cpu")
        qq = gen(synth.TAG_Q, 10, 0, 0, 512, 4, 64, 1.0, "cpu")
        ref = oracle_mod.attention(qq, np.arange(512), kk, vv, W)
        err = np.abs(o[0].float().cpu().double().numpy() - ref)
        out.append({"workload": f"swa_layer_512_W{W}_Hq4_Hkv1_d64", "metric": "latency", "unit": "us",
                    "value": round(ms * 1000, 2), "max_abs_err": float(err.max()), "mean_abs_err": float(err.mean())})

    # config 3: 16K chunk after a 131072-token prefix; SWA layer W=128 (ring) + full layer (pages)
    P, Nc, Hq, Hkv, d, W = 131072, 16384, 64, 8, 128, 128
    total = P + Nc
    pages = total // 64
    pool = hs.kv_pool_create(hs.PoolDesc(1, 1, W, Hkv, d, 1, pages))
    perm = synth.permutation(SEED, synth.stream_id(synth.TAG_MISC, 3), pages).to(torch.int32)
    pt = perm.view(1, pages).to(dev)
    sid = torch.zeros(1, dtype=torch.int32, device=dev)
    sp = torch.tensor([P], dtype=torch.int64, device=dev)
    kp = gen(synth.TAG_K, 0, 100, P - W, W, Hkv, d, 1.0, dev)[None]
    vp = gen(synth.TAG_V, 0, 100, P - W, W, Hkv, d, 1.0, dev)[None]
    hs.kv_pool_append(pool, 0, kp, vp, torch.tensor([P - W], device=dev), seq_ids=sid)
    for c0 in range(0, total, 16384):
        n = min(16384, total - c0)
        kf = gen(synth.TAG_K, 1, 100, c0, n, Hkv, d, 1.0, dev)[None]
        vf = gen(synth.TAG_V, 1, 100, c0, n, Hkv, d, 1.0, dev)[None]
        hs.kv_pool_append(pool, 1, kf, vf, torch.tensor([c0], device=dev), page_table=pt)
    q0 = gen(synth.TAG_Q, 0, 100, P, Nc, Hq, d, 1.0, dev)[None]
    k0 = gen(synth.TAG_K, 0, 100, P, Nc, Hkv, d, 1.0, dev)[None]
    v0 = gen(synth.TAG_V, 0, 100, P, Nc, Hkv, d, 1.0, dev)[None]
    q1 = gen(synth.TAG_Q, 1, 100, P, Nc, Hq, d, 1.0, dev)[None]
    o0 = torch.empty_like(q0)
    o1 = torch.empty_like(q1)
    ms_swa = t(lambda: hs.swa_prefill_fwd(pool, 0, q0, k0, v0, o=o0, start_pos=sp, seq_ids=sid), 20)
    ms_full = t(lambda: hs.full_prefill_fwd(pool, 1, q1, pt, o=o1, start_pos=sp), 3, warm=1)
    swa_flops = 4 * d * Nc * W * Hq
    swa_bytes = (2 * Nc * Hq * d + 2 * Nc * Hkv * d + 2 * W * Hkv * d) * 2
    full_flops = 4 * d * (Nc * P + Nc * (Nc + 1) // 2) * Hq
    rows = [0, 1, 127, 128, 8191, 16383]
    qq = gen(synth.TAG_Q, 0, 100, P, Nc, Hq, d, 1.0, "cpu")[rows]
    kk = gen(synth.TAG_K, 0, 100, P - W + 1, Nc + W - 1, Hkv, d, 1.0, "cpu")
    vv = gen(synth.TAG_V, 0, 100, P - W + 1, Nc + W - 1, Hkv, d, 1.0, "cpu")
    e_swa = np.abs(o0[0, rows].float().cpu().double().numpy() -
                   oracle_mod.attention(qq, P + np.array(rows), kk, vv, W, key_base=P - W + 1))
    rows_f = [0, 16383]
    qf = gen(synth.TAG_Q, 1, 100, P, Nc, Hq, d, 1.0, "cpu")[rows_f]
    kf = gen(synth.TAG_K, 1, 100, 0, total, Hkv, d, 1.0, "cpu")
    vf = gen(synth.TAG_V, 1, 100, 0, total, Hkv, d, 1.0, "cpu")
    e_full = np.abs(o1[0, rows_f].float().cpu().double().numpy() -
                    oracle_mod.attention(qf, P + np.array(rows_f), kf, vf, 0))
    out.append({"workload": "hybrid_chunk16k_after_131072_swa_W128_Hq64_Hkv8_d128", "metric": "KV+Q+O GB/s",
                "unit": "GB/s", "value": round(swa_bytes / ms_swa / 1e6, 1), "ms": round(ms_swa, 4),
                "tflops": round(swa_flops / ms_swa / 1e9, 1), "pct_hbm_peak": round(100 * swa_bytes / ms_swa / 1e6 / hbm, 1),
                "max_abs_err": float(e_swa.max()), "mean_abs_err": float(e_swa.mean())})
    out.append({"workload": "hybrid_chunk16k_after_131072_full_paged_Hq64_Hkv8_d128", "metric": "prefill TFLOP/s",
                "unit": "TFLOP/s", "value": round(full_flops / ms_full / 1e9, 1), "ms": round(ms_full, 3),
                "pct_bf16_peak": round(100 * full_flops / ms_full / 1e9 / bf16, 1),
                "max_abs_err": float(e_full.max()), "mean_abs_err": float(e_full.mean())})
    del pool, q0, k0, v0, q1, o0, o1
    torch.cuda.empty_cache()

    # config 4: decode batch
    out.extend(decode_results(hs, oracle_mod, hbm))
    # config 5: the 70-layer schedule on the last chunk of a 1M-token prefill
    if bf16_sus is not None:
        out.append(long_context_result(hs, oracle_mod, bf16_sus))
    return out


def decode_results(hs, oracle_mod, hbm, with_aux=True):
    res = decode_step_result(hs, oracle_mod, hbm, fp8=False)
    res += decode_step_result(hs, oracle_mod, hbm, fp8=True)
    if with_aux:
        res += aux_results(hs, oracle_mod)
    return res


def decode_step_result(hs, oracle_mod, hbm, fp8):
    """The hybrid decode step (7 calls) on a bf16 or an FP8 pool, L2 flushed before each step."""
    dev = "cuda"
    wl = DecodeBatch(hs, fp8=fp8)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(2):
        wl.step()
    torch.cuda.synchronize()
    times, times_full = [], []
    for _ in range(5):
        flush.zero_()
        ev = []
        a = torch.cuda.Event(True)
        a.record()
        wl.step(ev)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(ev[-1][1]))
        times_full.append(ev[-1][0].elapsed_time(ev[-1][1]))
    ms = statistics.median(times)
    ms_full = statistics.median(times_full)
    assert hs.hswa_pool_check_error(wl.pool) == 0
    mx, mean = wl.check_sample(oracle_mod)
    res = [{"workload": wl.name, "metric": "hybrid decode KV GB/s",
            "unit": "GB/s", "value": round(wl.bytes / ms / 1e6, 1), "ms": round(ms, 3),
            "pct_hbm_peak": round(100 * wl.bytes / ms / 1e6 / hbm, 1), "bytes": wl.bytes, "sum_ctx": wl.S,
            "full_layer_ms": round(ms_full, 3), "full_layer_gbs": round(wl.full_bytes_per_launch / ms_full / 1e6, 1),
            "kv_format": "fp8_e4m3" if fp8 else "bf16",
            "l2": "flushed (256 MiB write) before each step", "max_abs_err": mx, "mean_abs_err": mean}]
    del wl
    torch.cuda.empty_cache()
    return res


def aux_results(hs, oracle_mod):
    """window_safe_len over 4096 requests and the host prefix-cache match."""
    dev = "cuda"
    W = 128
    res = []
    # window_safe_len over 4096 requests (bit-exact vs oracle)
    nr = 4096
    C = synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 11), nr, 0, 262144)
    M = torch.where(synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 12), nr, 0, 1) == 0, C,
                    synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 13), nr, 0, 262144))
    # masks: half all-valid, a quarter with one random evicted slot, a quarter with slot C mod W evicted
    bits = np.full((nr, W // 32), 0xFFFFFFFF, dtype=np.uint32)
    ev = synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 14), nr, 0, W - 1).numpy()
    kind = synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 15), nr, 0, 3).numpy()
    for r in range(nr):
        s = int(C[r]) % W if kind[r] == 3 else (int(ev[r]) if kind[r] == 2 else -1)
        if s >= 0:
            bits[r, s // 32] &= np.uint32(~(1 << (s % 32)) & 0xFFFFFFFF)
    Md, Cd, Bd = M.to(dev), C.to(dev), torch.from_numpy(bits.view(np.int32)).to(dev)
    outw = torch.empty(nr, dtype=torch.int64, device=dev)
    for _ in range(5):
        hs.window_safe_len(Md, Cd, Bd, W, out=outw)
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(True), torch.cuda.Event(True)
    a.record()
    for _ in range(100):
        hs.window_safe_len(Md, Cd, Bd, W, out=outw)
    b_.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b_) / 100 * 1000
    ref = oracle_mod.window_safe_len(M.numpy(), C.numpy(), bits, W)
    res.append({"workload": "window_safe_len_4096req_W128", "metric": "latency", "unit": "us", "value": round(us, 2),
                "requests_per_s": round(nr / (us * 1e-6)), "bit_exact": bool(np.array_equal(outw.cpu().numpy(), ref))})
    res.append(prefix_cache_result(hs, oracle_mod))
    return res


def prefix_cache_result(hs, oracle_mod, nr=4096, W=128, max_len=2048):
    """SWA-aware prefix cache (host code): nr cached sequences of lengths C in [0, max_len] with
    their own tokens, evictions following the window_safe_len request recipe, then nr matches.
    With one sequence per path the window-safe length equals window_safe_len(m, C, mask), which
    the oracle computes in closed form (bit-exact check over every request)."""
    C = synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 21), nr, 0, max_len).numpy()
    M = np.where(synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 22), nr, 0, 1).numpy() == 0, C,
                 synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 23), nr, 0, max_len).numpy())
    ev = synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 24), nr, 0, W - 1).numpy()
    kind = synth.uniform_int(SEED, synth.stream_id(synth.TAG_MISC, 25), nr, 0, 3).numpy()
    bits = np.full((nr, W // 32), 0xFFFFFFFF, dtype=np.uint32)
    tree = hs.PrefixTree(W)
    seqs = []
    t0 = time.perf_counter()
    for r in range(nr):
        seq = np.arange(int(C[r]), dtype=np.int32) + np.int32(r * 65536)  # tokens of this sequence only
        seqs.append(seq)
        tree.insert(seq)
    t_insert = time.perf_counter() - t0
    for r in range(nr):
        s = int(C[r]) % W if kind[r] == 3 else (int(ev[r]) if kind[r] == 2 else -1)
        if s < 0:
            continue
        bits[r, s // 32] &= np.uint32(~(1 << (s % 32)) & 0xFFFFFFFF)
        for p in range(max(0, int(C[r]) - W), int(C[r])):  # the window position in that slot
            if p % W == s:
                tree.evict_swa(seqs[r], p, p + 1)
    queries = []
    for r in range(nr):
        k = min(int(M[r]), int(C[r]))
        extra = np.full(int(M[r]) - k, -1, dtype=np.int32)  # a token no cached sequence holds
        queries.append(np.concatenate([seqs[r][:k], extra]))
    times = []
    for _ in range(3):
        t0 = time.perf_counter()
        m_len, safe = tree.match_batch(queries)
        times.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    ref = oracle_mod.window_safe_len(M.astype(np.int64), C.astype(np.int64), bits, W)
    n_pos, n_held = tree.stats()
    tree.close()
    return {"workload": f"prefix_cache_match_{nr}req_W{W}_len{max_len}", "metric": "host match latency", "unit": "us",
            "value": round(sec * 1e6, 1), "requests_per_s": round(nr / sec), "matched_tokens": int(m_len.sum()),
            "ns_per_matched_token": round(sec * 1e9 / max(1, int(m_len.sum())), 1), "cached_positions": n_pos,
            "positions_holding_swa_kv": n_held, "insert_s": round(t_insert, 3),
            "bit_exact": bool(np.array_equal(safe, ref)), "where": "host CPU, one thread"}


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args, ws, rank):
    if rank != 0:
        return
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    B, N, W, Hq, Hkv, d = 2, 16384, 4096, 32, 8, 128
    sigma = 2 ** -0.5
    n_rows = 32
    rows = np.arange(N - n_rows, N)
    lo = rows[0] - W + 1
    k = gen(synth.TAG_K, 0, 0, lo, N - lo, Hkv, d, sigma, "cpu")
    v = gen(synth.TAG_V, 0, 0, lo, N - lo, Hkv, d, sigma, "cpu")
    q = gen(synth.TAG_Q, 0, 0, rows[0], n_rows, Hq, d, sigma, "cpu")
    for _ in range(args.warmup):
        oracle.attention(q, rows, k, v, W, key_base=lo, n_threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention(q, rows, k, v, W, key_base=lo, n_threads=threads)
    dt = (time.perf_counter() - t0) / args.steps
    flops = 4 * d * n_rows * W * Hq
    val = flops / dt / 1e12
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1000, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": SwaPrefill16k.config(ws, B, N, W, Hq, Hkv, d),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n_rows} query rows x {Hq} heads at the end of sequence 0 (full W-key windows) per step"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

# the sources each workload's dominant kernel is built from (a stored traffic figure stands while
# they are unchanged)
KERNEL_SOURCES = {
    "swa_prefill_16k": ["prefill_sm100.cu", "prefill_tile.cuh", "common.cuh", "internal.h"],
    "full_chunk_131k": ["prefill_sm100.cu", "prefill_tile.cuh", "common.cuh", "internal.h"],
    "long_context_1m": ["prefill_sm100.cu", "prefill_tile.cuh", "common.cuh", "internal.h"],
    "swa_chunk_131k": ["prefill_narrow.cu", "prefill_tile.cuh", "common.cuh", "internal.h"],
    "hybrid_decode": ["decode.cu", "decode_tc.cuh", "common.cuh", "internal.h"],
    "hybrid_decode_fp8": ["decode.cu", "decode_tc.cuh", "common.cuh", "internal.h"],
}


def kernel_source_sha(workload: str) -> str:
    """Hash of the CUDA sources of a workload's dominant kernel, to tell whether a stored ncu
    traffic figure still describes them."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hybrid_sliding_window_swa_b200", "csrc")
    for f in KERNEL_SOURCES[workload]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from profiles/traffic.json, or None when the
    kernel sources changed since that ncu capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f).get(workload)
        if d and d.get("source_sha") == kernel_source_sha(workload):
            return d["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="hswa", choices=["hswa", "reference"])
    ap.add_argument("--workload", default="swa_prefill_16k",
                    choices=["swa_prefill_16k", "long_context_1m", "hybrid_decode", "swa_chunk_131k",
                             "full_chunk_131k"])
    ap.add_argument("--decode-seqs", type=int, default=256, help="sequences in the hybrid_decode batch")
    ap.add_argument("--kv-format", default="bf16", choices=["bf16", "fp8"],
                    help="storage of the hybrid_decode pool's K/V entries")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads", "seqs"],
                    help="with several GPUs: replicas = every rank its own problem (weak scaling); heads = the "
                         "16K chunk split by KV head; seqs = the decode batch split by sequence (strong scaling)")
    ap.add_argument("--gather-o", action="store_true", help="--shard heads: all-gather O over NCCL every step")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    big = args.workload == "long_context_1m"
    if args.steps is None:
        args.steps = 5 if big else 20
    if args.warmup is None:
        args.warmup = 3 if big else 5
    args.warmup = max(args.warmup, 3)

    ws, rank, local = dist_setup() if args.impl == "hswa" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        run_reference(args, ws, rank)
        return

    torch.cuda.set_device(local)
    import hybrid_sliding_window_swa_b200 as hs
    hs.load_library()
    if args.shard == "heads" and args.workload != "swa_prefill_16k":
        raise SystemExit("--shard heads applies to the swa_prefill_16k workload")
    if args.shard == "seqs" and args.workload != "hybrid_decode":
        raise SystemExit("--shard seqs applies to the hybrid_decode workload")
    hbm, bf16, bf16_sus, peak_src = peaks()
    decode = args.workload in ("hybrid_decode", "swa_chunk_131k")  # bandwidth-bound: GB/s
    if args.workload in ("swa_chunk_131k", "full_chunk_131k"):
        wl = HybridChunk131k(hs, kind="swa" if args.workload == "swa_chunk_131k" else "full", seq_offset=rank,
                             fp8=args.kv_format == "fp8")
        dominant_flops = wl.flops
        if decode:
            peak, peak_name = hbm, f"{peak_src} HBM copy bandwidth"
        else:
            peak, peak_name = bf16, f"{peak_src} bf16 burst"
    elif big:
        wl = LongContext1M(hs, seq_offset=rank)
        dominant_flops = wl.full_flops_per_launch
        peak = bf16_sus  # a seconds-long step: the sustained figure
        peak_name = f"{peak_src} bf16 sustained"
    elif args.workload == "hybrid_decode":
        if args.shard == "seqs":
            ranks, _ = hs.hswa_shard_sequences(DecodeBatch.batch_lens(args.decode_seqs).numpy(), ws)
            wl = DecodeBatch(hs, n=args.decode_seqs, fp8=args.kv_format == "fp8",
                             select=np.nonzero(ranks == rank)[0])
        else:
            wl = DecodeBatch(hs, n=args.decode_seqs, seq_offset=rank, fp8=args.kv_format == "fp8")
        wl.flops = wl.bytes  # the decode metric counts bytes
        dominant_flops = wl.full_bytes_per_launch
        peak = hbm
        peak_name = f"{peak_src} HBM copy bandwidth"
    elif args.shard == "heads":
        wl = SwaPrefill16k(hs, heads=hs.hswa_shard_kv_heads(8, ws, rank), gather_o=args.gather_o)
        dominant_flops = wl.flops
        peak = bf16
        peak_name = f"{peak_src} bf16 burst"
    else:
        wl = SwaPrefill16k(hs, seq_offset=rank * 2)
        dominant_flops = wl.flops
        peak = bf16
        peak_name = f"{peak_src} bf16 burst"
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()
    assert hs.hswa_pool_check_error(wl.pool) == 0

    kern_events = []
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        wl.step(kern_events)
    e1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    kern_ms = sum(a.elapsed_time(b) for a, b in kern_events) / len(kern_events)
    ms_max = max_over_ranks(ms_step, ws)
    scale = 1e6 if decode else 1e9  # GB/s for the decode workload, TFLOP/s otherwise
    units_total = sum_over_ranks(wl.flops, ws)  # every rank's units (replicas: ws x one problem)
    value = units_total / ms_max / scale
    achieved = dominant_flops / kern_ms / scale
    assert hs.hswa_pool_check_error(wl.pool) == 0

    max_err, mean_err = (None, None)
    e2e = None
    cpu = None
    sec = None
    if not args.no_e2e and not big:
        wl.e2e_setup()
        e2e_begin = getattr(wl, "e2e_begin", lambda: None)
        e2e_end = getattr(wl, "e2e_end", lambda: None)
        e2e_begin()
        for _ in range(2):
            wl.e2e_step()
        e2e_end()
        torch.cuda.synchronize()
        barrier(ws)
        a, b = torch.cuda.Event(True), torch.cuda.Event(True)
        # a pipelined loop is timed over enough steps that its fill and drain (both inside the
        # timed region) do not dominate the per-step figure
        n_e2e = max(16, args.steps) if getattr(wl, "pipelined", False) else max(3, args.steps // 4)
        a.record()
        e2e_begin()
        for _ in range(n_e2e):
            wl.e2e_step()
        e2e_end()
        b.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, ws)
        e2e = {"value": round(units_total / e2e_ms / scale, 2), "unit": "GB/s" if decode else "TFLOP/s",
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h,
               "path": ("pinned host Q and new K/V of 7 layers -> device, 7 hybrid_decode_fwd calls via the Python "
                        "binding (C ABI), O of 7 layers -> pinned host") if args.workload == "hybrid_decode" else
                       ("pinned host Q/K/V -> device (copy stream), swa_prefill_fwd + kv_pool_append via the "
                        "Python binding (C ABI), O -> pinned host (second copy stream); consecutive steps overlap "
                        "on two device buffer sets") if args.workload == "swa_prefill_16k" else
                       "pinned host inputs of the chunk -> device, the attention call via the Python binding (C ABI), "
                       "O -> pinned host"}
    if rank == 0:
        import oracle
        oracle.build()
        max_err, mean_err = wl.check_sample(oracle)
        if not args.no_cpu:
            threads = os.cpu_count() or 1
            dt, fl, nrows = wl.oracle_sample(oracle, threads=threads)
            if args.workload == "hybrid_decode":
                cpu = {"value": fl / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                       "sample": f"all 4 x 64 rows of the {nrows} shortest sequences on the full layer, fp64, "
                                 f"{dt:.1f} s"}
            elif args.workload in ("swa_chunk_131k", "full_chunk_131k"):
                cpu = {"value": fl / dt / (1e9 if decode else 1e12), "unit": "GB/s" if decode else "TFLOP/s",
                       "cores": threads, "kind": "oracle",
                       "sample": f"{nrows} query rows x 64 heads of the layer, fp64, {dt:.1f} s"}
            else:
                what = ("32 heads at the end of sequence 0 (full 4096-key windows)" if not big else
                        "64 heads of SWA layer 3 (full 128-key windows)")
                cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                       "sample": f"{nrows} query rows x {what}, fp64, {dt:.1f} s"}
        if not args.no_secondary and ws == 1 and not big and not decode:
            sec = secondary_results(hs, oracle, hbm, bf16, bf16_sus)

    if rank == 0:
        if big:
            config = {"workload": wl.name, "B_per_gpu": 1, "seq_len": wl.N, "chunk": wl.Nc, "window": wl.W,
                      "Hq": wl.Hq, "Hkv": wl.Hkv, "head_dim": wl.d, "layers": "60 SWA + 10 full, interleaved 6:1",
                      "parallelism": f"independent sequences x{ws}", "step": "70 attention calls on the chunk",
                      "l2": "inputs larger than L2 (each full layer reads 4 GiB of pages)",
                      "footprint": wl.footprint()}
            kname = "prefill_kernel<128> (full_prefill_fwd, one full layer)"
        elif args.workload in ("swa_chunk_131k", "full_chunk_131k"):
            config = {"workload": wl.name, "B_per_gpu": 1, "prefix": wl.P, "chunk": wl.Nc,
                      "window": wl.W if wl.kind == "swa" else None, "Hq": wl.Hq, "Hkv": wl.Hkv, "head_dim": wl.d,
                      "parallelism": f"independent sequences x{ws}",
                      "step": "swa_prefill_fwd" if wl.kind == "swa" else "full_prefill_fwd (chunk appended first)",
                      "kv_format": "fp8_e4m3" if wl.fp8 else "bf16",
                      "l2": "inputs larger than L2"}
            kname = ("prefill_narrow_kernel<128> (swa_prefill_fwd, W <= 129 path)" if wl.kind == "swa" else
                     "prefill_kernel<128> (full_prefill_fwd)")
        elif decode:
            config = {"workload": wl.name, "n_seqs_per_gpu": wl.n, "sum_ctx": wl.S, "max_ctx": wl.maxL,
                      "tokens_per_seq": wl.nq, "window": wl.W, "Hq": wl.Hq, "Hkv": wl.Hkv, "head_dim": wl.d,
                      "kv_format": "fp8_e4m3" if wl.fp8 else "bf16",
                      "layers": "6 SWA (ring) + 1 full (pages)",
                      "parallelism": (f"sequences split over {ws} ranks (length buckets, longest first onto the "
                                      f"least-loaded rank; this rank {wl.n} sequences)" if args.shard == "seqs"
                                      else f"independent batches x{ws}"),
                      "step": "7 hybrid_decode_fwd calls", "bytes_per_step": wl.bytes,
                      "l2": "inputs larger than L2 (tens of GB of K/V per step)"}
            kname = ("hybrid_decode_fwd on the full layer (plan_kernel + decode_kernel<128,2> on FP8 blocks + "
                     "merge_kernel)" if wl.fp8
                     else "hybrid_decode_fwd on the full layer (plan_kernel + decode_kernel<128,2> + merge_kernel)")
        else:
            config = SwaPrefill16k.config(ws, wl.B, wl.N, wl.W, wl.Hq, wl.Hkv, wl.d, args.shard, args.gather_o)
            kname = "prefill_kernel<128> (swa_prefill_fwd)"
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s" if decode else "TFLOP/s", "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True,
            "scaling": "strong" if args.shard in ("heads", "seqs") else "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded counter-based normal, rounded to bf16)",
            "config": config,
            ("pct_hbm_peak" if decode else "pct_bf16_peak"): round(100 * value / ws / (hbm if decode else bf16), 1),
            "roofline": {"bound": "hbm" if decode else "tensor", "kernel": kname,
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s" if decode else "TFLOP/s",
                         "frac": round(achieved / peak, 3), "peak_source": peak_name,
                         ("algorithmic_bytes_per_launch" if decode else "algorithmic_flops_per_launch"): dominant_flops,
                         "kernel_ms": round(kern_ms, 4), "traffic": stored_traffic(args.workload + ("_fp8" if args.kv_format == "fp8" and decode else ""))},
            "parity": {"max_abs_err": max_err, "mean_abs_err": mean_err},
            "gpu_launches": wl.launches_per_step * args.steps,
            "clocks": clk,
        }
        if cpu:
            line["cpu_baseline"] = cpu
        if e2e:
            line["e2e"] = e2e
        elif big:
            line["e2e"] = None
            line["e2e_note"] = ("not measured for this workload: one step's inputs are 23 GB of host memory "
                                "(70 layers of Q plus the SWA chunks' K/V)")
        if sec:
            line["secondary"] = sec
        bad = []
        if not parity_ok(max_err, mean_err):
            bad.append(wl.name)
        for r in sec or []:
            if "max_abs_err" in r and not parity_ok(r["max_abs_err"], r["mean_abs_err"]):
                bad.append(r["workload"])
            if r.get("bit_exact") is False:
                bad.append(r["workload"])
        line["parity"]["ok"] = not bad
        if bad:
            line["parity"]["failed"] = bad
        print(json.dumps(line), flush=True)
    else:
        bad = []
    if ws > 1:
        torch.distributed.destroy_process_group()
    if bad:
        sys.stderr.write(f"parity check failed against the oracle: {bad}\n")
        sys.exit(1)


if __name__ == "__main__":
    main()
