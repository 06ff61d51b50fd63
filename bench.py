#!/usr/bin/env python
"""Benchmark of the MSA routed-memory hot path on B200 (libmsa).

Default workload: routed decode over a 100M-token memory bank on one GPU, 18 routed
layers (200,000 docs x 500 tokens -> 1,600,000 chunks of 64; K̄_r bf16 [chunks, 8, 128] per
layer resident in HBM, 3.28 GB per layer, 59 GB in total; K̄/V̄ bf16 in pinned host memory,
the selected documents fetched per layer), batch of 4 decode queries (T = 1, 32 query
heads, 8 KV heads, d = 128, k = 16, 2048-token local KV cache each).

One step = for each routed layer: route + top-k over the whole bank (msa_route_topk),
context assembly from the host bank (msa_fetch_begin/finish; copies overlap the next
layer's scan), sparse attention (msa_sparse_attend). Queries/s = B / step time.

``--workload bank10m`` runs the 10M-token single-layer decode (20,000 docs, B = 8, device
bank) instead. ``--workload prefill1m`` times the 1M-token prefill path (1,024 docs x 1,024
tokens: doc-wise RoPE + chunk pooling of K, V, K_r, bank preparation, tensor-core routing of a
128-token query, gather, attention) phase by phase; its line reports bank tokens/s.
``--workload interleave10m`` runs Memory Interleaving at its full configuration (18 routed
layers, each over its own 10M-token bank; B = 32 queries of T = 256 tokens, k = 8, 3 rounds:
each round re-routes with the appended documents excluded and attends over their raw K/V
placed before the query tokens); its line reports queries/s of the whole interleave.
``--workload attend_long`` times one msa_sparse_attend call alone at the last interleave round's
shape with 4 queries (256 tokens, 64 memory + 8,256 local rows): the small case for profiling
the tensor-core attention. ``--workload gen100m`` runs sparse generation at the 100M-token bank: per request the context is
built once (the default workload's step: 18 routed layers of route + host-bank gather +
attention of the query token), then 256 tokens are generated per query, each through 18
decode steps (msa_decode_step: the token's K/V appended to the layer's 2,048-row local cache,
attention over [gathered memory ; cache]); its line reports generated tokens/s.
``--workload encode_hidden1m`` times the offline encode from hidden states at the 1M-token bank
(1,024 docs x 1,024 tokens, hidden size 2,560: the three projections on tcgen05 fused with
doc-wise RoPE and chunk pooling). ``--impl reference`` times the CPU oracle on the host cores (a bounded
sample of the same workload). Under torchrun every rank runs an independent replica
(the path does not shard: no collective on the data path).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA routed-decode queries/s at 10M/100M-token bank; router-scan HBM GB/s"
UNIT = "queries/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libmsa", choices=["libmsa", "reference"])
    ap.add_argument("--workload", default="bank100m",
                    choices=["bank100m", "bank10m", "prefill1m", "interleave10m", "attend_long",
                             "gen100m", "encode_hidden1m", "attend_bwd", "fetch100m",
                             "aux_loss"])
    ap.add_argument("--gen-tokens", type=int, default=256,
                    help="gen100m: tokens generated per query after the context is built")
    ap.add_argument("--fetch", default="zerocopy", choices=["memcpy", "zerocopy"],
                    help="host-bank fetch: device gather over the host link on a side stream "
                         "(zerocopy) or host-issued cudaMemcpyAsync per selected run (memcpy)")
    ap.add_argument("--scan", default="tc", choices=["tc", "cc"],
                    help="router scan: tensor cores over the normalised bank, or CUDA cores")
    ap.add_argument("--cached", action="store_true",
                    help="routed decode: keep each layer's local K/V as a rotated cache that the "
                         "step appends the query token to (msa_decode_step) instead of passing it "
                         "before RoPE to msa_sparse_attend every step")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels one by one instead of replaying a CUDA graph")
    ap.add_argument("--layers", type=int, default=0,
                    help="routed decode (bank100m, bank10m): routed layers per step (0: the "
                         "configuration's; one layer of the 100M-token bank is the 3.3 GB case "
                         "the DRAM counters are captured on)")
    ap.add_argument("--docs", type=int, default=0,
                    help="encode_hidden1m: documents of 1,024 tokens (0: the configuration's "
                         "1,024; fewer make the small case the kernel's counters are captured on)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-layers", type=int, default=3,
                    help="routed layers in the CPU-oracle sample")
    return ap.parse_args()


def captured_traffic(kernel_srcs, summary: str):
    """DRAM bytes (read + write) of one launch from a committed ncu capture, or None when the
    kernel's sources changed since the capture (the summary records the SHA-256 of the
    sources concatenated in the order given)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", summary)) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for src in kernel_srcs:
            with open(os.path.join(ROOT, "long_context_doc_b200", "csrc", src), "rb") as f:
                h.update(f.read())
        if rec.get("kernel_src_sha256") != h.hexdigest():
            return None
        return int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"])
    except Exception:
        return None


def peaks():
    """HBM roofline denominator: the measured STREAM-style copy bandwidth (reads and writes
    together), else the pool's earlier fallback figure. A pure read stream can run a little
    above a copy, so a read-only kernel may show a fraction slightly above 1."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured copy (read+write)"
    except Exception:
        return 6650.0, "fallback copy (read+write)"


HBM_NOMINAL_GBS = 7700.0  # HGX B200 HBM3e, for context beside the measured copy peak


# ------------------------------------------------------------------------------ ranks
class Ranks:
    """One process per GPU (torchrun's RANK / WORLD_SIZE / LOCAL_RANK; rendezvous on
    MASTER_ADDR, 127.0.0.1 on one node). The path does not shard: every rank runs its own
    replica, and the only collectives are the timing barrier and the max over ranks of the
    measured times."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: int = 300):
        import torch.distributed as dist
        self.dist = dist
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" and device is not None else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, values, device):
        """Element-wise max over ranks of a list of floats (every rank gets the result)."""
        if self.world == 1:
            return [float(v) for v in values]
        import torch
        t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return [float(v) for v in t.tolist()]

    def close(self):
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()


def replica_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Whole-job throughput of ``world`` replicas that each processed ``units_per_rank`` in at
    most ``ms`` milliseconds (the max over ranks)."""
    return world * units_per_rank / (ms / 1e3)


def queue_ahead(stream, ms: float = 20.0):
    """Hold ``stream`` in a GPU spin of about ``ms`` milliseconds (cycles at up to 2 GHz) so
    that the eager launches made after it are queued before the GPU reaches them: the CUDA
    events placed between them then time device work alone, with no host launch gap inside."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(ms * 2e6))


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summarize(self.lines)

    @classmethod
    def summarize(cls, lines):
        """Median SM clock, the highest max clock and the throttle reasons seen active, from
        ``nvidia-smi --format=csv,noheader,nounits`` lines of FIELDS (malformed lines skipped)."""
        sm, mx, reasons = [], [], set()
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(cls.NAMES, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ workload
class Decode:
    """The routed decode workload: synthetic banks and queries fed to the package's
    ``engine.RoutedDecode`` (per layer route -> fetch/gather -> attend; see its docstring for
    the overlapped schedule)."""

    def __init__(self, w, dev, fetch: str, rank: int, scan: str = "tc", nbuf: int = 2,
                 cached: bool = False):
        import torch

        import long_context_doc_b200 as msa
        import synth
        from long_context_doc_b200.engine import DecodeLayer, RoutedDecode
        self.torch, self.msa, self.w, self.dev = torch, msa, w, dev
        # the 10M-token bank keeps K̄/V̄ in HBM; the 100M-token bank's live in pinned host memory
        fetch = fetch if w.n_docs * w.doc_len > 50_000_000 else "device"
        self.L = w.layers
        self.scan = scan
        self.cached = cached
        seed_w = w.scaled(seed=w.seed + 1000 * rank)
        B = w.B
        # every layer's query inputs in one contiguous buffer: first the router queries Q_r of
        # all layers (what the routing reads), then per layer Q and, with caches, the token's K/V
        # (what only the attention reads), so that a step's host copy is two transfers and the
        # second can go in beside the routing
        nqr, nq = B * w.T * w.h_qr * w.d, B * w.T * w.h_q * w.d
        nkv = B * w.T * w.h_kv * w.d if cached else 0
        self.n_route_in = self.L * nqr
        att_per_layer = nq + 2 * nkv
        self.qbuf = torch.empty(self.n_route_in + self.L * att_per_layer, dtype=torch.bfloat16,
                                device=dev)
        # rotated local caches of L_loc rows: the first L_loc - 1 hold the prompt, the step
        # appends the query token's own K/V; a step starts by resetting every length
        self.lens = torch.zeros(self.L, dtype=torch.int32, device=dev)
        self.lens0 = torch.full((self.L,), w.L_loc - w.T, dtype=torch.int32, device=dev)
        Kh = Vh = None
        coff_host = None
        layers = []
        for l in range(self.L):
            dv = synth.dev_bank_workload(seed_w, dev, layer=l, with_kv=(fetch == "device"))
            coff_host = dv["doc_chunk_off"]
            if fetch != "device" and Kh is None:
                Kh, Vh = self._host_bank(seed_w, coff_host, dev)
            base = self.n_route_in + l * att_per_layer
            Q_r = self.qbuf[l * nqr:(l + 1) * nqr].view(dv["Q_r"].shape)
            Q = self.qbuf[base:base + nq].view(dv["Q"].shape)
            Q_r.copy_(dv["Q_r"])
            Q.copy_(dv["Q"])
            kv = (Kh, Vh) if fetch != "device" else (dv["Kbar"], dv["Vbar"])
            if scan == "tc":
                # the tensor-core scan reads only the normalised bank: K̄_r is not kept
                rkw = dict(Kbar_r_hat=msa.kr_normalize(dv.pop("Kbar_r")))
            else:
                rkw = dict(Kbar_r=dv["Kbar_r"], kr_inv_norm=msa.kr_inv_norm(dv["Kbar_r"]))
            if cached:
                T = w.T
                c = msa.LocalCache(B, w.L_loc, w.h_kv, w.d, pos0=w.k, rope_base=w.rope_base,
                                   device=dev, length=self.lens[l:l + 1])
                c.append(dv["K_loc"][:, :-T].contiguous(), dv["V_loc"][:, :-T].contiguous())
                o = base + nq
                K_new = self.qbuf[o:o + nkv].view(B, T, w.h_kv, w.d)
                V_new = self.qbuf[o + nkv:o + 2 * nkv].view(B, T, w.h_kv, w.d)
                K_new.copy_(dv["K_loc"][:, -T:])
                V_new.copy_(dv["V_loc"][:, -T:])
                la = DecodeLayer(Q_r, Q, None, None, kv[0], kv[1], cache=c, K_new=K_new,
                                 V_new=V_new, **rkw)
            else:
                la = DecodeLayer(Q_r, Q, dv["K_loc"], dv["V_loc"], kv[0], kv[1], **rkw)
            layers.append(la)
            del dv
        self.rd = RoutedDecode(layers, coff_host, w.k, w.rope_base, fetch=fetch, nbuf=nbuf)
        self.fetch = self.rd.fetch
        self.main = self.rd.stream
        self.layers = layers
        self.n_chunks = self.rd.n_chunks
        self.max_ctx = self.rd.max_ctx
        self.obuf = self.rd.O.view(-1)
        self.kernels_per_step = self.rd.kernels_per_step()

    @staticmethod
    def _host_bank(w, coff_host, dev):
        """One pinned host K̄/V̄ bank shared by the routed layers (only the selected rows ever
        cross the host link, so the fetch traffic does not depend on this)."""
        import torch

        import synth
        n_chunks = int(coff_host[-1])
        Kh = torch.empty((n_chunks, w.h_kv, w.d), dtype=torch.bfloat16, pin_memory=True)
        Vh = torch.empty_like(Kh, pin_memory=True)
        tmp = torch.empty((1 << 20, w.h_kv, w.d), dtype=torch.bfloat16, device=dev)
        row = w.h_kv * w.d
        for tid, dst in ((synth.KBAR, Kh), (synth.VBAR, Vh)):
            for c0 in range(0, n_chunks, tmp.shape[0]):
                n = min(tmp.shape[0], n_chunks - c0)
                t = tmp[:n]
                synth.dev_normal(t, w.seed, synth.tag(tid, 0), first=c0 * row)
                dst[c0:c0 + n].copy_(t)
        del tmp
        return Kh, Vh

    @property
    def route_ev(self):
        return self.rd.route_events

    @route_ev.setter
    def route_ev(self, ev):
        self.rd.route_events = ev

    def step(self, local_ready=None):
        import torch
        if self.cached:  # every cache back to its prompt; the step appends the token
            with torch.cuda.stream(self.main):
                self.lens.copy_(self.lens0)
        self.rd.step(local_ready)

    def ctx(self, l):
        """(ctxK, ctxV, ctx_len) of layer l after a step (with one buffer set per layer)."""
        bf = self.rd.buf[l % self.rd.nbuf]
        return bf["cK"], bf["cV"], self.rd.ctx_len[l]

    def scan_bytes(self):
        """Algorithmic bytes of one routing call: the bank it streams (K̂_r for the tensor
        path; K̄_r plus fp32 inverse norms for the CUDA-core path)."""
        w = self.w
        if self.scan == "tc":
            return self.n_chunks * w.h_kv * w.d * 2
        return self.n_chunks * w.h_kv * w.d * 2 + self.n_chunks * w.h_kv * 4


def run_libmsa(args):
    import torch

    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    rank, world = ranks.rank, ranks.world
    w = synth.C4 if args.workload == "bank100m" else synth.C3
    if args.layers > 0 and args.layers != w.layers:
        w = w.scaled(layers=args.layers, name=w.name.replace(f"_{w.layers}l", "") +
                     f"_{args.layers}l")
    wk = Decode(w, dev, args.fetch, rank, args.scan, cached=args.cached)
    torch.cuda.synchronize()

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        wk.step()
    barrier()
    # the step as one CUDA graph (the zero-copy and device fetches need no host round trip)
    use_graph = not args.no_graph and wk.fetch != "memcpy"
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=wk.main):
            wk.step()
    barrier()

    def run_step():
        if graph is not None:
            with torch.cuda.stream(wk.main):  # replay on the stream the timing events use
                graph.replay()
        else:
            wk.step()

    run_step()
    barrier()

    Kst = args.steps
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(Kst - 1)]  # between steps
    barrier()
    t0.record(wk.main)
    for s in range(Kst):
        run_step()
        if s + 1 < Kst:
            marks[s].record(wk.main)
    t1.record(wk.main)
    barrier()
    clocks = sampler.stop()
    step_ms = t0.elapsed_time(t1) / Kst
    bounds = [t0] + marks + [t1]
    per_step = sorted(bounds[i].elapsed_time(bounds[i + 1]) for i in range(Kst))
    step_dist = {"p10": round(float(np.percentile(per_step, 10)), 4),
                 "median": round(float(np.percentile(per_step, 50)), 4),
                 "p90": round(float(np.percentile(per_step, 90)), 4)}
    # routing-call durations for the roofline: the same step launched eagerly with CUDA events
    # around every msa_route_topk call (on the launching stream), the launches queued ahead of
    # the GPU so that the events time the call's kernels and not the host's launch latency
    Kr = max(3, min(Kst, 20))
    ev_route = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(wk.L)] for _ in range(Kr)]
    queue_ahead(wk.main)  # the eager launches queue up behind a spin: no host gap in a call
    with torch.cuda.stream(wk.main):
        for s in range(Kr):
            wk.route_ev = ev_route[s]
            wk.step()
    barrier()
    wk.route_ev = None
    route_ms = [ev_route[s][l][0].elapsed_time(ev_route[s][l][1])
                for s in range(Kr) for l in range(wk.L)]
    # end to end: per-step query inputs copied from pinned host memory, outputs read back
    # per step: every layer's Q_r and Q (one copy), the new token's K/V row of every layer's
    # local cache, then every layer's output (one copy) and every layer's top-k ids (one copy)
    host_q = wk.qbuf.cpu().pin_memory()  # every layer's Q_r, Q (and the token's K/V if cached)
    host_kv = ([] if wk.cached else
               [[t.cpu().pin_memory() for t in (d.K_loc[:, -1:], d.V_loc[:, -1:])]
                for d in wk.layers])
    host_O = wk.obuf.cpu().pin_memory()
    host_ids = wk.rd.ids.cpu().pin_memory()
    h2d = (host_q.numel() * host_q.element_size() +
           sum(t.numel() * t.element_size() for hs in host_kv for t in hs))
    d2h = host_O.numel() * host_O.element_size() + host_ids.numel() * 4

    kv_stream = torch.cuda.Stream(dev)
    att_ready, step_done = torch.cuda.Event(), torch.cuda.Event()
    nr = wk.n_route_in

    def e2e_step():
        with torch.cuda.stream(wk.main):
            wk.qbuf[:nr].copy_(host_q[:nr], non_blocking=True)  # the router queries
        # what only the attention reads (Q, the new token's K/V) goes in on a side stream while
        # the first layers route; the previous step's attention, which read it, comes before
        kv_stream.wait_stream(wk.main)
        with torch.cuda.stream(kv_stream):
            wk.qbuf[nr:].copy_(host_q[nr:], non_blocking=True)
            for l in range(len(host_kv)):
                d = wk.layers[l]
                kn, vn = host_kv[l]
                d.K_loc[:, -1:].copy_(kn, non_blocking=True)
                d.V_loc[:, -1:].copy_(vn, non_blocking=True)
            att_ready.record(kv_stream)
        with torch.cuda.stream(wk.main):
            wk.step(att_ready)
            step_done.record(wk.main)
            host_O.copy_(wk.obuf, non_blocking=True)
        # the two reads back run side by side
        kv_stream.wait_event(step_done)
        with torch.cuda.stream(kv_stream):
            host_ids.copy_(wk.rd.ids, non_blocking=True)
        wk.main.wait_stream(kv_stream)

    for _ in range(3):
        e2e_step()
    barrier()
    e_graph = None
    if use_graph:
        e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e_graph, stream=wk.main):
            e2e_step()
        with torch.cuda.stream(wk.main):
            e_graph.replay()
        barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    Ke = max(5, Kst // 2)
    e0.record(wk.main)
    for _ in range(Ke):
        if e_graph is not None:
            with torch.cuda.stream(wk.main):
                e_graph.replay()
        else:
            e2e_step()
    e1.record(wk.main)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / Ke
    step_ms, e2e_ms = ranks.max([step_ms, e2e_ms], dev)  # max over ranks
    value = replica_rate(world, w.B, step_ms)
    e2e_value = replica_rate(world, w.B, e2e_ms)
    route_avg = statistics.mean(route_ms)
    peak, peak_kind = peaks()
    achieved = wk.scan_bytes() / (route_avg / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": Kst,
        "warmup": max(args.warmup, 3), "ms_per_step": round(step_ms, 4),
        "step_ms_dist": step_dist,  # per timed step (rank 0), CUDA events between the steps
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 normals, planted docs; no dataset)",
        "config": {"workload": w.name, "bank_tokens": w.n_docs * w.doc_len, "n_docs": w.n_docs,
                   "n_chunks": wk.n_chunks, "chunk": w.chunk, "routed_layers": wk.L,
                   "batch": w.B, "T": w.T, "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d, "k": w.k,
                   "local_kv": w.L_loc,
                   "kv_bank": ("pinned host memory, one K̄/V̄ bank shared by the routed layers, "
                               f"fetch={wk.fetch}") if wk.fetch != "device" else "HBM",
                   "l2": "no flush: every layer scans a 3.28 GB K̄_r, far larger than the 126 MB L2"
                   if wk.L > 1 else "no flush: the 328 MB K̄_r scan exceeds the 126 MB L2",
                   "scan": wk.scan, "cuda_graph": use_graph,
                   "local_kv_form": ("rotated cache: the step appends the query token's K/V "
                                     "(RoPE at pos0 + 2047) to a 2047-row cache and attends "
                                     "(msa_decode_step)") if wk.cached else
                                    "K_loc before RoPE, all 2048 keys rotated per step "
                                    "(msa_sparse_attend)",
                   "parallelism": f"replicas x{world}"},
        "router_scan_gbs": round(achieved, 1),
        "roofline": {"kernel": ("msa_route_topk (tensor-core scan: query fold + tcgen05 scan + "
                               "document top-k)" if wk.scan == "tc" else
                               "msa_route_topk (CUDA-core scan with fused top-k)"), "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "frac_of_nominal": round(achieved / HBM_NOMINAL_GBS, 4),
                     "traffic": (captured_traffic(("route_tc.cu", "common.cuh"),
                                                   f"route_tc_{w.name}_dram.json")
                                 if wk.scan == "tc" else None),
                     "bytes_per_launch": wk.scan_bytes(),
                     "avg_launch_ms": round(route_avg, 4),
                     "timing": "CUDA events around every routing call of an eager pass of the "
                               "same step after the timed replays, its launches queued behind "
                               "a GPU spin (no host launch gap inside a call)"},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": Kst * wk.kernels_per_step,
        "route_calls_timed": len(route_ms),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_layers)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, e_graph  # graphs are released before the process group
    ranks.close()


# ------------------------------------------------------------------------------ CPU oracle
def oracle_layer_time(w, layer: int) -> float:
    """Oracle time of one routed layer of the decode workload for the whole batch:
    route over every document, gather, attend (inputs generated beforehand, untimed)."""
    import oracle
    import synth
    inp = synth.make_bank_workload(w, layer, with_bank=False)
    coff = inp["doc_chunk_off"]
    Krb = synth.host_bank_rows(w, "Kbar_r", 0, int(coff[-1]), layer=layer, coff=coff,
                               Q_r=inp["Q_r"])
    t0 = time.perf_counter()
    ids, _, _ = oracle.route(inp["Q_r"], Krb, coff, w.k)
    max_ctx = w.k * int(np.max(np.diff(coff)))
    gi, cl = oracle.gather(ids, coff, max_ctx)
    t1 = time.perf_counter()
    del Krb
    # the gathered rows only (the oracle reads bank rows through the gather indices)
    rows = np.unique(gi[gi >= 0])
    remap = np.full(int(coff[-1]), -1, np.int64)
    remap[rows] = np.arange(len(rows))
    Kb = np.concatenate([synth.host_bank_rows(w, "Kbar", int(r), int(r) + 1, layer=0)
                         for r in rows])
    Vb = np.concatenate([synth.host_bank_rows(w, "Vbar", int(r), int(r) + 1, layer=0)
                         for r in rows])
    gi2 = np.where(gi >= 0, remap[np.maximum(gi, 0)], -1).astype(np.int32)
    t2 = time.perf_counter()
    oracle.attend(inp["Q"], inp["K_loc"], inp["V_loc"], Kb, Vb, gi2, cl, w.k, w.rope_base)
    t3 = time.perf_counter()
    return (t1 - t0) + (t3 - t2)


def cpu_baseline(w, n_layers: int) -> dict:
    import oracle
    times = [oracle_layer_time(w, l) for l in range(n_layers)]
    per_layer = sum(times) / len(times)
    step = per_layer * w.layers
    return {"value": round(w.B / step, 4), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"{n_layers} of {w.layers} routed layers of the same workload, each: route "
                       f"over all {w.n_docs} docs + gather + attend for the batch of {w.B}; "
                       f"step time = mean layer time x {w.layers}"),
            "cpu_seconds": round(sum(times), 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synth
    if args.workload == "gen100m":
        w = synth.C4
        # each timed step = 4 generation steps of ONE routed layer (a bounded sample); the
        # tokens/s extrapolate its mean per-token time to all routed layers
        times = []
        for s in range(args.steps):
            times.append(oracle_generate_time(w, s % w.layers, 4))
            if sum(times) > 120:
                break
        sample = statistics.mean(times)
        token = sample / 4 * w.layers
        value = w.B / token
        unit = "generated tokens/s"
        print(json.dumps({
            "metric": "MSA sparse generation tokens/s at the 100M-token bank (context built once "
                      "per request, routed memory fixed while generating)",
            "value": round(value, 4), "unit": unit, "n_gpus": 1, "steps": len(times),
            "warmup": args.warmup, "ms_per_step": round(sample * 1e3, 2),
            "step_is": f"4 generation steps of one routed layer of {w.layers} (value = batch / "
                       f"(mean step time / 4 x {w.layers}))",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "gen100m", "routed_layers": w.layers, "batch": w.B,
                       "prompt_local_kv": w.L_loc},
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "kind": "oracle",
                             "cores": oracle.num_threads(),
                             "sample": "each step = 4 generation steps of one routed layer for "
                                       "the batch x the layer count (construction left out)"},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return
    w = synth.C4 if args.workload == "bank100m" else synth.C3
    for l in range(min(args.warmup, 1)):
        oracle_layer_time(w.scaled(n_docs=2000), l)
    # each timed step is a bounded sample of the workload's step: ONE routed layer (route over
    # every document + gather + attend for the batch); the queries/s extrapolate it to all
    # routed layers, while steps and ms_per_step describe what was actually timed
    times = []
    for s in range(args.steps):
        times.append(oracle_layer_time(w, s % w.layers))
        if sum(times) > 60:
            break
    layer = statistics.mean(times)
    value = w.B / (layer * w.layers)
    line = {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": 1,
            "steps": len(times), "warmup": args.warmup, "ms_per_step": round(layer * 1e3, 2),
            "step_is": f"one routed layer of {w.layers} (value = batch / ({w.layers} x mean "
                       "layer time))",
            "extrapolated_ms_per_full_step": round(layer * w.layers * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "bank_tokens": w.n_docs * w.doc_len,
                       "routed_layers": w.layers, "batch": w.B, "k": w.k},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "kind": "oracle",
                             "cores": oracle.num_threads(),
                             "sample": "each timed step = one routed layer (route over every "
                                       "doc + gather + attend for the batch); value "
                                       "extrapolates the mean layer time to all routed layers"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill(args):
    """The 1M-token prefill path, each phase timed with CUDA events on the launching stream."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev, timeout_s=300)
    rank, world = ranks.rank, ranks.world
    w = synth.C2.scaled(seed=synth.C2.seed + 1000 * rank)
    inp = synth.dev_token_workload(w, dev)
    off = inp["doc_tok_off"]
    n_tok = int(off[-1])
    n_chunks = msa.msa_count_chunks(off, w.chunk)
    cpd = max(-(-int(off[i + 1] - off[i]) // w.chunk) for i in range(w.n_docs))
    max_ctx = w.k * cpd
    bf = torch.bfloat16
    Kb = torch.empty((n_chunks, w.h_kv, w.d), dtype=bf, device=dev)
    Vb, Rb, hat = torch.empty_like(Kb), torch.empty_like(Kb), torch.empty_like(Kb)
    inv = torch.empty((n_chunks, w.h_kv), dtype=torch.float32, device=dev)
    coff = torch.empty(w.n_docs + 1, dtype=torch.int64, device=dev)
    tok_off = torch.from_numpy(np.ascontiguousarray(off, dtype=np.int64)).to(dev)
    ws_r = torch.empty(msa.msa_route_topk_workspace(w.B, w.T, w.h_qr, w.h_kv, w.d, 1, w.n_docs,
                                                    n_chunks, w.k), dtype=torch.uint8, device=dev)
    ids = torch.empty((w.B, w.k), dtype=torch.int32, device=dev)
    sc = torch.empty((w.B, w.k), dtype=torch.float32, device=dev)
    gi = torch.empty((w.B, max_ctx), dtype=torch.int32, device=dev)
    cl = torch.empty(w.B, dtype=torch.int32, device=dev)
    cK = torch.empty((w.B, max_ctx, w.h_kv, w.d), dtype=bf, device=dev)
    cV = torch.empty_like(cK)
    ws_g = torch.zeros(256, dtype=torch.uint8, device=dev)
    ws_a = torch.empty(msa.msa_sparse_attend_workspace(w.B, w.T, w.h_q, w.h_kv, w.d, max_ctx,
                                                       w.L_loc), dtype=torch.uint8, device=dev)
    O = torch.empty((w.B, w.T, w.h_q, w.d), dtype=bf, device=dev)
    st = torch.cuda.Stream()
    names = ["encode_pool", "kr_normalize", "route_topk", "gather", "sparse_attend"]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]

    def step(rec):
        if rec:
            ev[0].record(st)
        msa.msa_encode_pool(inp["K"], inp["V"], inp["K_r"], off, tok_off, w.chunk, w.rope_base,
                            Kb, Vb, Rb, inv, coff, st)
        if rec:
            ev[1].record(st)
        msa.msa_kr_normalize(Rb, hat, st)
        if rec:
            ev[2].record(st)
        msa.msa_route_topk(inp["Q_r"], Rb, inv, coff, w.k, None, ids, sc, None, ws_r, st, hat)
        if rec:
            ev[3].record(st)
        msa.msa_gather(ids, coff, Kb, Vb, max_ctx, gi, cl, cK, cV, ws_g, st)
        if rec:
            ev[4].record(st)
        msa.msa_sparse_attend(inp["Q"], inp["K_loc"], inp["V_loc"], cK, cV, cl, w.k, w.rope_base,
                              0.0, O, ws_a, st)
        if rec:
            ev[5].record(st)

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        step(False)
    barrier()
    Kst = max(1, min(args.steps, 20))
    phase = {n: [] for n in names}
    totals = []
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    for _ in range(Kst):
        queue_ahead(st, 5.0)  # the step's launches queue up behind a spin: device time alone
        step(True)
        st.synchronize()
        for i, n in enumerate(names):
            phase[n].append(ev[i].elapsed_time(ev[i + 1]))
        totals.append(ev[0].elapsed_time(ev[-1]))
    clocks = sampler.stop()
    step_ms = statistics.mean(totals)
    step_ms, = ranks.max([step_ms], dev)  # max over ranks
    ph = {n: round(statistics.mean(v), 4) for n, v in phase.items()}
    peak, peak_kind = peaks()
    row = w.h_kv * w.d * 2
    enc_bytes = 3 * n_tok * row + 3 * n_chunks * row + n_chunks * w.h_kv * 4
    enc_gbs = enc_bytes / (ph["encode_pool"] / 1e3) / 1e9
    route_bytes = n_chunks * row
    line = {
        "metric": "MSA 1M-token prefill: bank tokens/s (doc-wise RoPE + pooling, routing, "
                  "gather, attention)",
        "value": round(replica_rate(world, n_tok, step_ms), 1), "unit": "bank tokens/s",
        "n_gpus": world, "steps": Kst, "warmup": max(args.warmup, 3),
        "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 normals, planted docs; no dataset)",
        "config": {"workload": w.name, "bank_tokens": n_tok, "n_docs": w.n_docs,
                   "n_chunks": n_chunks, "chunk": w.chunk, "batch": w.B, "T": w.T,
                   "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d, "k": w.k, "local_kv": w.L_loc,
                   "l2": "no flush: the encode reads 6.4 GB per step, 51x the 126 MB L2",
                   "launch": "eager; each timed step's launches queued behind a short GPU spin, "
                             "so its events time device work and no host launch gap",
                   "parallelism": f"replicas x{world}"},
        "phases_ms": ph,
        "roofline": {"kernel": "msa_encode_pool (doc-wise RoPE + chunk mean of K, V, K_r)",
                     "bound": "hbm", "achieved": round(enc_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(enc_gbs / peak, 4), "peak_kind": peak_kind, "traffic": None,
                     "bytes_per_launch": enc_bytes, "avg_launch_ms": ph["encode_pool"]},
        "route_scan_gbs": round(route_bytes / (ph["route_topk"] / 1e3) / 1e9, 1),
        "gpu_launches": Kst * 8,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def run_interleave(args):
    """Memory Interleaving at full size, each phase timed with CUDA events on its stream."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev, timeout_s=600)
    rank, world = ranks.rank, ranks.world
    w = synth.C5.scaled(seed=synth.C5.seed + 1000 * rank)
    B, T, k, R, NL = w.B, w.T, w.k, w.rounds, w.layers
    bf = torch.bfloat16
    lay = []
    for l in range(NL):
        d = synth.dev_bank_workload(w, dev, layer=l, with_kv=True)
        d["inv"] = msa.kr_inv_norm(d["Kbar_r"])
        d["hat"] = msa.kr_normalize(d["Kbar_r"])
        lay.append(d)
    coff_host = lay[0]["doc_chunk_off"]
    coff = torch.from_numpy(coff_host).to(dev)
    n_chunks, n_docs = int(coff_host[-1]), w.n_docs
    max_ctx = k * int(np.max(np.diff(coff_host)))
    words = (n_docs + 31) // 32
    # raw per-token K/V of appended documents: a per-layer pool of P synthetic documents
    # (document d uses pool entry d mod P; the content does not change the cost)
    P = 16
    pools = []
    for l in range(NL):
        kp = torch.empty((P, w.doc_len, w.h_kv, w.d), dtype=bf, device=dev)
        vp = torch.empty_like(kp)
        synth.dev_normal(kp, w.seed, synth.tag(synth.APPK, l))
        synth.dev_normal(vp, w.seed, synth.tag(synth.APPV, l))
        pools.append((kp, vp))
    Ls = [T + r * k * w.doc_len for r in range(R)]
    kloc = [None] + [torch.empty((B, Lr, w.h_kv, w.d), dtype=bf, device=dev) for Lr in Ls[1:]]
    vloc = [None] + [torch.empty_like(t) for t in kloc[1:]]
    doc_bytes = w.doc_len * w.h_kv * w.d * 2
    seglen = [None] + [torch.full((B, r * k), w.doc_len, dtype=torch.int32, device=dev)
                       for r in range(1, R)]
    ws_s = torch.zeros(256, dtype=torch.uint8, device=dev)
    ws_r = torch.empty(msa.msa_route_topk_workspace(B, T, w.h_qr, w.h_kv, w.d, 1, n_docs,
                                                    n_chunks, k), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(max(msa.msa_sparse_attend_workspace(B, T, w.h_q, w.h_kv, w.d, max_ctx, Lr)
                           for Lr in Ls), dtype=torch.uint8, device=dev)
    ids = torch.empty((B, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, k), dtype=torch.float32, device=dev)
    gi = torch.empty((B, max_ctx), dtype=torch.int32, device=dev)
    cl = torch.empty(B, dtype=torch.int32, device=dev)
    cK = torch.empty((B, max_ctx, w.h_kv, w.d), dtype=bf, device=dev)
    cV = torch.empty_like(cK)
    ws_g = torch.zeros(256, dtype=torch.uint8, device=dev)
    O = torch.empty((B, T, w.h_q, w.d), dtype=bf, device=dev)
    appended = torch.zeros((B, R * k), dtype=torch.int64, device=dev)
    excl = torch.zeros((B, words), dtype=torch.int64, device=dev)
    ex32 = torch.zeros((B, words), dtype=torch.int32, device=dev)
    st = torch.cuda.Stream()
    names = ["route", "gather", "assemble", "attend"]
    nev = R * NL
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(nev)]
    rows_b = torch.arange(B, device=dev).unsqueeze(1)

    def interleave(rec):
        with torch.cuda.stream(st):
            excl.zero_()
            for r in range(R):
                A = r * k * w.doc_len
                for l in range(NL):
                    ev = evs[r * NL + l]
                    d = lay[l]
                    if rec:
                        ev[0].record(st)
                    msa.msa_route_topk(d["Q_r"], d["Kbar_r"], d["inv"], coff, k,
                                       ex32 if r > 0 else None, ids, sc, None, ws_r, st,
                                       d["hat"])
                    if rec:
                        ev[1].record(st)
                    msa.msa_gather(ids, coff, d["Kbar"], d["Vbar"], max_ctx, gi, cl, cK, cV,
                                   ws_g, st)
                    if rec:
                        ev[2].record(st)
                    if r > 0:  # [appended documents (round order, ascending id) ; query tokens]
                        idx = (appended[:, :r * k] % P) * doc_bytes
                        msa.msa_assemble_local(idx + pools[l][0].data_ptr(),
                                               idx + pools[l][1].data_ptr(), seglen[r],
                                               d["K_loc"], d["V_loc"], kloc[r], vloc[r], ws_s, st)
                        kl, vl = kloc[r], vloc[r]
                    else:  # round 0: the query tokens alone
                        kl, vl = d["K_loc"], d["V_loc"]
                    if rec:
                        ev[3].record(st)
                    msa.msa_sparse_attend(d["Q"], kl, vl, cK, cV, cl, k, w.rope_base, 0.0, O,
                                          ws_a, st)
                    if rec:
                        ev[4].record(st)
                # the last routed layer's documents are appended and excluded from now on
                new = torch.sort(ids.to(torch.int64), dim=1).values
                appended[:, r * k:(r + 1) * k] = new
                excl.scatter_add_(1, new // 32, torch.ones_like(new) << (new % 32))
                ex32.copy_(excl.to(torch.int32))

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    for _ in range(max(1, min(args.warmup, 2))):
        interleave(False)
    barrier()
    Kst = max(1, min(args.steps, 3))
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    phase = {n: 0.0 for n in names}
    per_round_attend = [0.0] * R
    per_round_route = [0.0] * R
    t0.record(st)
    for _ in range(Kst):
        interleave(True)
        st.synchronize()
        for r in range(R):
            for l in range(NL):
                ev = evs[r * NL + l]
                for i, n in enumerate(names):
                    phase[n] += ev[i].elapsed_time(ev[i + 1]) / Kst
                per_round_attend[r] += ev[3].elapsed_time(ev[4]) / Kst
                per_round_route[r] += ev[0].elapsed_time(ev[1]) / Kst
    t1.record(st)
    barrier()
    clocks = sampler.stop()
    step_ms = t0.elapsed_time(t1) / Kst
    step_ms, = ranks.max([step_ms], dev)  # max over ranks
    route_flop = 2.0 * B * T * n_chunks * w.h_kv * w.d  # per routing call
    route_call_ms = phase["route"] / (R * NL)
    route_tf = route_flop / (route_call_ms / 1e3) / 1e12
    # attention: QK^T and PV over the visible keys (memory rows + causal local rows)
    att_flop = 0.0
    for r in range(R):
        vis = max_ctx + Ls[r] - T + (T + 1) / 2.0
        att_flop += NL * 4.0 * B * T * w.h_q * vis * w.d
    att_tf = att_flop / (phase["attend"] / 1e3) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        tpeak, tkind = float(pk["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        tpeak, tkind = 1410.0, "fallback (sustained)"
    line = {
        "metric": "MSA Memory Interleaving queries/s (18 routed layers x 3 rounds, 10M-token "
                  "bank per layer)",
        "value": round(replica_rate(world, B, step_ms), 3), "unit": "queries/s", "n_gpus": world,
        "steps": Kst, "warmup": max(1, min(args.warmup, 2)), "ms_per_step": round(step_ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 normals; appended documents from a per-layer pool)",
        "config": {"workload": w.name, "bank_tokens_per_layer": n_docs * w.doc_len,
                   "n_chunks": n_chunks, "routed_layers": NL, "rounds": R, "batch": B, "T": T,
                   "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d, "k": k, "local_kv_per_round": Ls,
                   "l2": "no flush: every layer reads its own 328 MB bank and 0.3-1 GB of K/V",
                   "parallelism": f"replicas x{world}"},
        "phases_ms": {n: round(v, 3) for n, v in phase.items()},
        "route_ms_per_round": [round(x, 3) for x in per_round_route],
        "attend_ms_per_round": [round(x, 3) for x in per_round_attend],
        "roofline": {"kernel": "msa_route_topk (tcgen05 scan, 8,192 query rows per call)",
                     "bound": "tensor", "achieved": round(route_tf, 1), "peak": tpeak,
                     "unit": "TFLOP/s", "frac": round(route_tf / tpeak, 4), "peak_kind": tkind,
                     "traffic": None, "flop_per_launch": route_flop,
                     "avg_launch_ms": round(route_call_ms, 4)},
        "attend_tflops": round(att_tf, 1),
        "gpu_launches": Kst * R * NL * 9,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def run_attend_long(args):
    """One long-query attention call (the last interleave round's shape, B = 4), CUDA events."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.C5
    B, T, L, mc = 4, w.T, w.T + 2 * w.k * w.doc_len, w.k * 8
    bf = torch.bfloat16
    Q = synth.dev_normal(torch.empty((B, T, w.h_q, w.d), dtype=bf, device=dev), w.seed, 1)
    Kl = synth.dev_normal(torch.empty((B, L, w.h_kv, w.d), dtype=bf, device=dev), w.seed, 2)
    Vl = synth.dev_normal(torch.empty_like(Kl), w.seed, 3)
    cK = synth.dev_normal(torch.empty((B, mc, w.h_kv, w.d), dtype=bf, device=dev), w.seed, 4)
    cV = synth.dev_normal(torch.empty_like(cK), w.seed, 5)
    cl = torch.full((B,), mc, dtype=torch.int32, device=dev)
    ws = torch.empty(msa.msa_sparse_attend_workspace(B, T, w.h_q, w.h_kv, w.d, mc, L),
                     dtype=torch.uint8, device=dev)
    O = torch.empty((B, T, w.h_q, w.d), dtype=bf, device=dev)
    st = torch.cuda.Stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(max(args.warmup, 3)):
        msa.msa_sparse_attend(Q, Kl, Vl, cK, cV, cl, w.k, w.rope_base, 0.0, O, ws, st)
    Kst = max(1, min(args.steps, 20))
    e0.record(st)
    for _ in range(Kst):
        msa.msa_sparse_attend(Q, Kl, Vl, cK, cV, cl, w.k, w.rope_base, 0.0, O, ws, st)
    e1.record(st)
    st.synchronize()
    ms = e0.elapsed_time(e1) / Kst
    flop = 4.0 * B * T * w.h_q * (mc + L - T + (T + 1) / 2.0) * w.d
    print(json.dumps({"metric": "long-query attention TFLOP/s (call incl. the RoPE pre-pass)",
                      "value": round(flop / (ms / 1e3) / 1e12, 1), "unit": "TFLOP/s",
                      "ms_per_call": round(ms, 4), "steps": Kst, "dtype": "bf16",
                      "config": {"workload": "attend_long", "batch": B, "T": T, "h_q": w.h_q,
                                 "h_kv": w.h_kv, "d": w.d, "memory_rows": mc, "local_rows": L}}),
          flush=True)


FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 148 SMs x 128 fp32 lanes x FMA at 1965 MHz


def run_aux_loss(args):
    """The auxiliary routing loss with its gradients (msa_aux_routing_loss: the chunk scores and
    their maximising tokens, the per-query loss and dL/ds, dK̄_r, dQ_r) over the 1M-token prefill
    bank (16,384 chunks of 8 KV heads x 128), B = 4 training queries of 128 tokens with 8 router
    heads, the chunks of 16 documents relevant per query; CUDA events on the launching stream,
    the calls queued behind a GPU spin."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.C2
    B, T = 4, w.T
    cpd = (w.doc_len + w.chunk - 1) // w.chunk
    n_chunks = w.n_docs * cpd
    bf = torch.bfloat16
    Q_r = synth.dev_normal(torch.empty((B, T, w.h_qr, w.d), dtype=bf, device=dev), w.seed, 11)
    K_r = synth.dev_normal(torch.empty((n_chunks, w.h_kv, w.d), dtype=bf, device=dev), w.seed, 12)
    words = (n_chunks + 31) // 32
    pos = np.zeros((B, words), np.uint32)
    rng = np.random.default_rng(w.seed)
    for b in range(B):  # the chunks of 16 relevant documents per query
        for doc in rng.choice(w.n_docs, 16, replace=False):
            for c in range(int(doc) * cpd, (int(doc) + 1) * cpd):
                pos[b, c // 32] |= np.uint32(1) << np.uint32(c % 32)
    bits = torch.from_numpy(pos.view(np.int32)).to(dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dQ = torch.empty((B, T, w.h_qr, w.d), dtype=torch.float32, device=dev)
    dK = torch.empty((n_chunks, w.h_kv, w.d), dtype=torch.float32, device=dev)
    ws_bytes = int(msa.lib.msa_aux_routing_loss_workspace(B, n_chunks))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream()
    for _ in range(max(args.warmup, 3)):
        msa.msa_aux_routing_loss(Q_r, K_r, bits, 0.1, loss, dQ, dK, ws, st)
    st.synchronize()
    assert np.isfinite(float(loss.item()))
    Kst = max(1, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    queue_ahead(st, 5.0)
    e0.record(st)
    for _ in range(Kst):
        msa.msa_aux_routing_loss(Q_r, K_r, bits, 0.1, loss, dQ, dK, ws, st)
    e1.record(st)
    st.synchronize()
    ms = e0.elapsed_time(e1) / Kst
    flop = 2.0 * B * T * w.h_qr * w.d * n_chunks  # the cosines' dot products (the bulk)
    tf = flop / (ms / 1e3) / 1e12
    cpu = None if args.no_cpu_baseline else cpu_aux_loss_baseline(w, B, T, n_chunks, flop)
    print(json.dumps({
        "metric": "auxiliary routing loss with gradients, TFLOP/s of the chunk-score cosines",
        "value": round(tf, 2), "unit": "TFLOP/s", "ms_per_call": round(ms, 4), "steps": Kst,
        "dtype": "bf16 in, f32 arithmetic",
        "config": {"workload": "aux_loss", "batch": B, "T": T, "h_qr": w.h_qr, "h_kv": w.h_kv,
                   "d": w.d, "n_chunks": n_chunks, "relevant_docs_per_query": 16, "tau": 0.1},
        "roofline": {"kernel": "msa_aux_routing_loss (4 launches: scores, loss, dK, dQ)",
                     "bound": "alu", "achieved": round(tf, 2),
                     "peak": round(FP32_ALU_TFLOPS, 1), "unit": "TFLOP/s",
                     "frac": round(tf / FP32_ALU_TFLOPS, 4),
                     "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 at 1965 MHz",
                     "traffic": None},
        "cpu_baseline": cpu}), flush=True)


def cpu_aux_loss_baseline(w, B: int, T: int, n_chunks: int, flop: float,
                          n_sample: int = 512) -> dict:
    """The oracle's auxiliary loss with its gradients on a bank of ``n_sample`` chunks (the same
    queries' shape, 16 relevant documents' worth of positives scaled down), its time scaled to
    the full bank by the chunk count (the oracle is linear in it)."""
    import oracle
    import synth
    Q = synth.normal(w.seed, 11, (B, T, w.h_qr, w.d), "bf16")
    K = synth.normal(w.seed, 12, (n_sample, w.h_kv, w.d), "bf16")
    pos = np.zeros((B, n_sample), bool)
    rng = np.random.default_rng(w.seed)
    for b in range(B):
        pos[b, rng.choice(n_sample, max(1, n_sample // 64), replace=False)] = True
    t0 = time.perf_counter()
    oracle.aux_routing_loss(synth.as_f32(Q, "bf16"), synth.as_f32(K, "bf16"), pos, 0.1)
    dt = time.perf_counter() - t0
    full = dt * n_chunks / n_sample
    return {"value": round(flop / full / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"the same call on {n_sample} of {n_chunks} chunks, time scaled by the "
                       f"chunk count ({dt:.2f} s measured, {full:.1f} s per full call)")}


def run_attend_backward(args):
    """The backward of the sparse attention at the last interleave round's shape (B = 4 queries
    of T = 256 tokens, 32 query heads over 8 KV heads, 64 memory rows + 8,256 local rows):
    msa_sparse_attend_backward (forward recompute, D, the tcgen05 gradient kernel, dQ rotated
    back) plus the scatter of the memory rows' gradients into an fp32 bank gradient, timed with
    CUDA events on the launching stream; TFLOP/s of the five backward products over the
    visible (query row, key) pairs."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev, timeout_s=300)
    rank, world = ranks.rank, ranks.world
    w = synth.C5
    B, T, L, mc = 4, w.T, w.T + 2 * w.k * w.doc_len, w.k * 8
    bf, f32 = torch.bfloat16, torch.float32
    seed = w.seed + 1000 * rank
    Q = synth.dev_normal(torch.empty((B, T, w.h_q, w.d), dtype=bf, device=dev), seed, 1)
    Kl = synth.dev_normal(torch.empty((B, L, w.h_kv, w.d), dtype=bf, device=dev), seed, 2)
    Vl = synth.dev_normal(torch.empty_like(Kl), seed, 3)
    cK = synth.dev_normal(torch.empty((B, mc, w.h_kv, w.d), dtype=bf, device=dev), seed, 4)
    cV = synth.dev_normal(torch.empty_like(cK), seed, 5)
    dO = synth.dev_normal(torch.empty_like(Q), seed, 6)
    cl = torch.full((B,), mc, dtype=torch.int32, device=dev)
    n_chunks = 20000 * 8
    gi = torch.stack([torch.randperm(n_chunks, device=dev)[:mc] for _ in range(B)]).to(torch.int32)
    g = dict(dQ=torch.empty((B, T, w.h_q, w.d), dtype=f32, device=dev),
             dK_loc=torch.empty((B, L, w.h_kv, w.d), dtype=f32, device=dev),
             dV_loc=torch.empty((B, L, w.h_kv, w.d), dtype=f32, device=dev),
             dK_ctx=torch.empty((B, mc, w.h_kv, w.d), dtype=f32, device=dev),
             dV_ctx=torch.empty((B, mc, w.h_kv, w.d), dtype=f32, device=dev))
    dKb = torch.zeros((n_chunks, w.h_kv, w.d), dtype=f32, device=dev)
    dVb = torch.zeros_like(dKb)
    ws = torch.empty(msa.msa_sparse_attend_backward_workspace(B, T, w.h_q, w.h_kv, w.d, mc, L),
                     dtype=torch.uint8, device=dev)
    ws_s = torch.zeros(256, dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream()

    def step():
        msa.msa_sparse_attend_backward(Q, Kl, Vl, cK, cV, cl, w.k, w.rope_base, 0.0, dO, g["dQ"],
                                       g["dK_loc"], g["dV_loc"], g["dK_ctx"], g["dV_ctx"], ws, st)
        msa.msa_scatter_bank_grad(gi, cl, g["dK_ctx"], g["dV_ctx"], dKb, dVb, ws_s, st)

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        step()
    barrier()
    assert msa.msa_workspace_status(ws, st) == 0
    Kst = max(1, min(args.steps, 20))
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(st)
    for _ in range(Kst):
        step()
    e1.record(st)
    barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / Kst
    ms, = ranks.max([ms], dev)
    # visible pairs: every row sees the memory rows and local rows up to L - T + t
    pairs = B * w.h_q * sum(mc + L - T + t + 1 for t in range(T))
    flop = 5 * 2.0 * pairs * w.d  # dP = dO V^T, dV = P^T dO, dK = dS^T Q, dQ = dS K (+ S again)
    sustained = 1410.6
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            sustained = float(json.load(f)["bf16_tflops_sustained"])
        kind = "measured (sustained)"
    except Exception:
        kind = "fallback (sustained)"
    tflops = flop / (ms / 1e3) / 1e12
    # end to end: inputs from pinned host memory, gradients read back, per step
    hQ, hK, hV, hc, hd = (t.cpu().pin_memory() for t in (Q, Kl, Vl, cK, dO))
    houts = {k: v.cpu().pin_memory() for k, v in g.items() if k in ("dQ", "dK_loc", "dV_loc")}
    h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV, hc, hd)) + hc.numel() * 2
    d2h = sum(t.numel() * t.element_size() for t in houts.values())

    def e2e_step():
        with torch.cuda.stream(st):
            for dst, src in ((Q, hQ), (Kl, hK), (Vl, hV), (cK, hc), (cV, hc), (dO, hd)):
                dst.copy_(src, non_blocking=True)
            step()
            for k, h in houts.items():
                h.copy_(g[k], non_blocking=True)

    e2e_step()
    barrier()
    Ke = max(3, Kst // 2)
    e0.record(st)
    for _ in range(Ke):
        e2e_step()
    e1.record(st)
    barrier()
    e_ms = e0.elapsed_time(e1) / Ke
    e_ms, = ranks.max([e_ms], dev)
    line = {
        "metric": "MSA sparse-attention backward TFLOP/s (5 products over the visible pairs; "
                  "forward recompute and bank scatter inside the timed call)",
        "value": round(replica_rate(world, tflops, 1e3), 1), "unit": "TFLOP/s", "n_gpus": world,
        "steps": Kst, "warmup": max(args.warmup, 3), "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normals)",
        "config": {"workload": "attend_bwd", "batch": B, "T": T, "h_q": w.h_q, "h_kv": w.h_kv,
                   "d": w.d, "memory_rows": mc, "local_rows": L,
                   "l2": "no flush: the local K/V read per call (135 MB) exceeds the 126 MB L2"},
        "roofline": {"kernel": "msa_sparse_attend_backward (whole call)", "bound": "tensor",
                     "achieved": round(tflops, 1), "peak": sustained, "unit": "TFLOP/s",
                     "frac": round(tflops / sustained, 4), "peak_kind": kind, "traffic": None,
                     "flop_per_call": flop},
        "e2e": {"value": round(replica_rate(world, flop / 1e12, e_ms), 1), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4)},
        "gpu_launches": Kst * 8,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def run_fetch(args):
    """The host-bank fetch of the 100M-token bank decode, measured on its own and beside the
    routing scan it overlaps: one routed layer (1.6M chunks), B = 4 queries, k = 16, the
    selected documents' K̄/V̄ rows (16 docs x 8 chunks x 2 KB, K and V) read from pinned host
    memory by (a) the zero-copy gather kernel on a side stream, (b) msa_fetch_begin/finish
    (one cudaMemcpyAsync per run of consecutive selected chunks). CUDA events on the
    launching streams; one JSON line."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.C4
    dv = synth.dev_bank_workload(w, dev, layer=0, with_kv=False)
    hat = msa.kr_normalize(dv.pop("Kbar_r"))
    coff_h = dv["doc_chunk_off"]
    coff = torch.from_numpy(coff_h).to(dev)
    n_chunks = int(coff_h[-1])
    Kh, Vh = Decode._host_bank(w, coff_h, dev)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    B, k = w.B, w.k
    max_ctx = k * int(np.max(np.diff(coff_h)))
    ws_r = torch.empty(msa.msa_route_topk_workspace(B, 1, w.h_qr, w.h_kv, w.d, 1, w.n_docs,
                                                    n_chunks, k), dtype=torch.uint8, device=dev)
    ids = torch.empty((B, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, k), dtype=torch.float32, device=dev)
    gi = torch.empty((B, max_ctx), dtype=torch.int32, device=dev)
    cl = torch.empty(B, dtype=torch.int32, device=dev)
    cK = torch.empty((B, max_ctx, w.h_kv, w.d), dtype=torch.bfloat16, device=dev)
    cV = torch.empty_like(cK)
    ws_g = torch.zeros(256, dtype=torch.uint8, device=dev)
    fetcher = msa.Fetcher(B, k)

    def route(st):
        msa.msa_route_topk(dv["Q_r"], None, None, coff, k, None, ids, sc, None, ws_r, st, hat)

    def gather(st):
        msa.msa_gather(ids, coff, Kh, Vh, max_ctx, gi, cl, cK, cV, ws_g, st)

    def memcpy_fetch(st):
        fetcher.begin(ids, coff, max_ctx, gi, cl, ws_g, st)
        fetcher.finish(coff_h, Kh, Vh, max_ctx, cK, cV, st, side, 10_000)

    def timed(fn, st, n=20):
        out = []
        for _ in range(n):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn(st)
            e1.record(st)
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1))
        return statistics.median(out)

    for _ in range(3):
        route(main)
        gather(main)
        memcpy_fetch(main)
    torch.cuda.synchronize()
    n_rows = int(cl.sum().item())
    row = w.h_kv * w.d * 2
    fetch_bytes = 2 * n_rows * row
    # runs of consecutive selected chunks (one cudaMemcpyAsync each, for K and for V)
    runs = 0
    for b in range(B):
        g = gi[b, :int(cl[b])].cpu().numpy()
        runs += int(1 + np.count_nonzero(np.diff(g) != 1)) if len(g) else 0
    t_route = timed(route, main)
    t_gather = timed(gather, side)
    t_memcpy = timed(memcpy_fetch, main)

    # routing with the fetch of another layer's selection running beside it on the side stream
    def route_with(fetch_fn):
        out = []
        for _ in range(20):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            fetch_fn()
            e0.record(main)
            route(main)
            e1.record(main)
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1))
        return statistics.median(out)

    def gather_side():
        gather(side)

    def memcpy_side():  # the copies go to the side stream; the ids are already on the host
        fetcher.begin(ids, coff, max_ctx, gi, cl, ws_g, side)
        fetcher.finish(coff_h, Kh, Vh, max_ctx, cK, cV, side, side, 10_000)

    t_route_zc = route_with(gather_side)
    t_route_mc = route_with(memcpy_side)
    line = {"metric": "host-bank fetch of the 100M-token bank decode (one routed layer, B = 4)",
            "workload": "fetch100m", "fetch_bytes": fetch_bytes, "context_rows": n_rows,
            "memcpy_runs": runs, "route_ms": round(t_route, 4),
            "zerocopy_gather": {"ms": round(t_gather, 4),
                                "gbs": round(fetch_bytes / (t_gather / 1e3) / 1e9, 2),
                                "route_ms_beside": round(t_route_zc, 4)},
            "memcpy_fetch": {"ms": round(t_memcpy, 4),
                             "gbs": round(fetch_bytes / (t_memcpy / 1e3) / 1e9, 2),
                             "copies": 2 * runs, "route_ms_beside": round(t_route_mc, 4)},
            "note": "memcpy ms spans msa_fetch_begin (gather indices + ids to the host) through "
                    "the copies and the event the main stream waits on, host wait included"}
    print(json.dumps(line), flush=True)
    fetcher.close()


def run_generate(args):
    """Sparse generation at the 100M-token bank: context construction once per request, then
    ``--gen-tokens`` decode steps through all routed layers; generated tokens/s."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev, timeout_s=300)
    rank, world = ranks.rank, ranks.world
    w = synth.C4
    if args.layers > 0 and args.layers != w.layers:
        w = w.scaled(layers=args.layers, name=w.name.replace(f"_{w.layers}l", "") +
                     f"_{args.layers}l")
    G = max(1, args.gen_tokens)
    # one context buffer per layer: the gathered memory stays fixed while tokens are generated
    wk = Decode(w, dev, args.fetch, rank, args.scan, nbuf=w.layers)
    B, L0, bf = w.B, w.L_loc, torch.bfloat16
    cap = L0 + G
    lens = torch.zeros(wk.L, dtype=torch.int32, device=dev)
    lens0 = torch.full((wk.L,), L0, dtype=torch.int32, device=dev)
    caches, tok = [], []
    ws_bytes = msa.msa_decode_step_workspace(B, 1, w.h_q, w.h_kv, w.d, wk.max_ctx, cap)
    # the generated token's query and K/V of every layer, in one contiguous buffer so that a
    # token's inputs arrive with a single host-to-device copy (synthetic, reused every step)
    nq, nkv = B * w.h_q * w.d, B * w.h_kv * w.d
    per_layer = nq + 2 * nkv
    tokbuf = torch.empty(wk.L * per_layer, dtype=bf, device=dev)
    for l in range(wk.L):
        c = msa.LocalCache(B, cap, w.h_kv, w.d, pos0=w.k, rope_base=w.rope_base, device=dev,
                           length=lens[l:l + 1])
        c.append(wk.layers[l].K_loc, wk.layers[l].V_loc)  # the prompt's local K/V
        caches.append(c)
        base = l * per_layer
        x = dict(Q=tokbuf[base:base + nq].view(B, 1, w.h_q, w.d),
                 K=tokbuf[base + nq:base + nq + nkv].view(B, 1, w.h_kv, w.d),
                 V=tokbuf[base + nq + nkv:base + per_layer].view(B, 1, w.h_kv, w.d),
                 O=torch.empty((B, 1, w.h_q, w.d), dtype=bf, device=dev),
                 ws=torch.empty(ws_bytes, dtype=torch.uint8, device=dev))
        for name, tid in (("Q", synth.GEN_Q), ("K", synth.GEN_K), ("V", synth.GEN_V)):
            synth.dev_normal(x[name], w.seed, synth.tag(tid, l))
        tok.append(x)
    torch.cuda.synchronize()
    assert int(lens[0]) == L0

    def token_step(rest_ready=None):
        for l in range(wk.L):
            if l == 1 and rest_ready is not None:  # the inputs of layers 1.. arrive beside layer 0
                wk.main.wait_event(rest_ready)
            x, c = tok[l], caches[l]
            cK, cV, cl = wk.ctx(l)
            msa.msa_decode_step(x["Q"], x["K"], x["V"], c.K, c.V, c.length, cK, cV, cl, w.k,
                                w.rope_base, 0.0, x["O"], x["ws"], wk.main)

    def construct():
        lens.copy_(lens0)  # a new request: every cache holds the prompt again
        wk.step()

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    with torch.cuda.stream(wk.main):
        for _ in range(max(args.warmup, 3)):
            construct()
            for _ in range(4):
                token_step()
    barrier()
    use_graph = not args.no_graph and wk.fetch != "memcpy"
    g_con = g_tok = None
    if use_graph:
        g_con, g_tok = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_con, stream=wk.main):
            construct()
        with torch.cuda.graph(g_tok, stream=wk.main):
            token_step()
    barrier()

    def request(ev=None):
        with torch.cuda.stream(wk.main):
            if g_con is not None:
                g_con.replay()
            else:
                construct()
            if ev is not None:
                ev.record(wk.main)
            for _ in range(G):
                if g_tok is not None:
                    g_tok.replay()
                else:
                    token_step()

    request()
    barrier()
    assert int(lens[0]) == cap and int(lens[-1]) == cap
    for l in range(wk.L):
        assert msa.msa_workspace_status(tok[l]["ws"], wk.main) == 0
    Kst = max(1, args.steps)
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(Kst)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(Kst)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(Kst)]
    barrier()
    t0.record(wk.main)
    for s in range(Kst):
        starts[s].record(wk.main)
        request(mids[s])
        ends[s].record(wk.main)
    t1.record(wk.main)
    barrier()
    clocks = sampler.stop()
    req_ms = t0.elapsed_time(t1) / Kst
    con_ms = statistics.mean(starts[s].elapsed_time(mids[s]) for s in range(Kst))
    tok_ms = statistics.mean(mids[s].elapsed_time(ends[s]) for s in range(Kst)) / G
    # decode-step duration for the roofline: the graph-replayed token step (18 routed layers,
    # each one msa_decode_step: append, attention, merge) divided by the layer count, so no
    # host launch gap enters it
    dec_avg = tok_ms / wk.L
    n_ev = G
    # algorithmic bytes of one decode step at the mean cache length of a request: memory
    # and local K/V rows read once, the query read, the output written, the token's K/V
    # appended (read + written)
    cl_host = [wk.rd.ctx_len[l].cpu().numpy() for l in range(wk.L)]
    mem_rows = statistics.mean(float(c.sum()) for c in cl_host)
    loc_rows = B * (L0 + (n_ev + 1) / 2.0)
    row = w.h_kv * w.d * 2
    step_bytes = ((mem_rows + loc_rows) * 2 * row + 2 * B * w.h_q * w.d * 2 + 4 * B * row)
    achieved = step_bytes / (dec_avg / 1e3) / 1e9
    # end to end: each token's per-layer inputs copied from pinned host memory and the last
    # layer's output read back, per generated token; the request's query inputs as in the
    # default workload
    host_tok = tokbuf.cpu().pin_memory()  # every layer's token inputs, one copy per token
    host_out = tok[-1]["O"].cpu().pin_memory()
    host_q = wk.qbuf.cpu().pin_memory()  # every layer's Q_r and Q of the request
    tok_h2d = host_tok.numel() * host_tok.element_size()
    q_h2d = host_q.numel() * host_q.element_size()
    h2d = q_h2d + G * tok_h2d
    d2h = G * host_out.numel() * host_out.element_size()

    tok_stream = torch.cuda.Stream(dev)
    rest_ready = torch.cuda.Event()

    def e2e_token():
        # layer 0's token inputs first; those of the other layers on a side stream while layer
        # 0 attends (the previous token's steps, which read them, come before)
        tokbuf[:per_layer].copy_(host_tok[:per_layer], non_blocking=True)
        ready = None
        if wk.L > 1:
            tok_stream.wait_stream(wk.main)
            with torch.cuda.stream(tok_stream):
                tokbuf[per_layer:].copy_(host_tok[per_layer:], non_blocking=True)
                rest_ready.record(tok_stream)
            ready = rest_ready
        token_step(ready)
        host_out.copy_(tok[-1]["O"], non_blocking=True)

    def e2e_con():
        wk.qbuf.copy_(host_q, non_blocking=True)
        construct()

    e_con = e_tok = None
    with torch.cuda.stream(wk.main):
        e2e_con()
        e2e_token()
    barrier()
    if use_graph:
        e_con, e_tok = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(e_con, stream=wk.main):
            e2e_con()
        with torch.cuda.graph(e_tok, stream=wk.main):
            e2e_token()
    barrier()
    Ke = max(1, min(Kst, 3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(wk.main)
    with torch.cuda.stream(wk.main):
        for _ in range(Ke):
            e_con.replay() if e_con is not None else e2e_con()
            for _ in range(G):
                e_tok.replay() if e_tok is not None else e2e_token()
    e1.record(wk.main)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / Ke
    req_ms, e2e_ms = ranks.max([req_ms, e2e_ms], dev)  # max over ranks
    unit = "generated tokens/s"
    value = replica_rate(world, B * G, req_ms)
    peak, peak_kind = peaks()
    line = {
        "metric": "MSA sparse generation tokens/s at the 100M-token bank (context built once per "
                  "request, routed memory fixed while generating)",
        "value": round(value, 1), "unit": unit, "n_gpus": world, "steps": Kst,
        "warmup": max(args.warmup, 3), "ms_per_step": round(req_ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 normals, planted docs; no dataset)",
        "config": {"workload": "gen100m" if wk.L == 18 else f"gen100m_{wk.L}l",
                   "bank_tokens": w.n_docs * w.doc_len,
                   "routed_layers": wk.L, "batch": B, "prompt_local_kv": L0,
                   "generated_tokens_per_query": G, "cache_capacity": cap, "k": w.k,
                   "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d,
                   "kv_bank": f"pinned host memory, fetch={wk.fetch}",
                   "l2": "no flush: the construction scans 18 x 3.28 GB; a token step reads 18 "
                         "layers' caches and memory (~40 MB each), 0.7 GB in total, above the "
                         "126 MB L2",
                   "cuda_graph": use_graph, "parallelism": f"replicas x{world}"},
        "construct_ms": round(con_ms, 3), "token_step_ms": round(tok_ms, 4),
        "roofline": {"kernel": "msa_decode_step (decode attention with the cache append fused "
                               "in + merge), per routed layer of the graph-replayed token step",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": captured_traffic(("attend_dec_plain.cu", "attend_dec.cu",
                                                  "common.cuh"),
                                                 "attend_dec_plain_gen100m_dram.json"),
                     "bytes_per_launch": round(step_bytes), "avg_launch_ms": round(dec_avg, 4)},
        "e2e": {"value": round(replica_rate(world, B * G, e2e_ms), 1), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 3)},
        # per request: the construction step's kernels + per token and layer the attention
        # (with the token's append) and the merge
        "gpu_launches": Kst * (wk.kernels_per_step + G * wk.L * 2),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_generate_baseline(w, G, args.cpu_layers)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_con, g_tok, e_con, e_tok
    ranks.close()


def oracle_generate_time(w, layer: int, steps: int) -> float:
    """Oracle time of ``steps`` generation steps of one routed layer for the whole batch
    (attention over 128 memory rows + the growing local context)."""
    import oracle
    import synth
    B, L0 = w.B, w.L_loc
    Kp = synth.normal(w.seed, synth.tag(synth.KLOC, layer), (B, L0, w.h_kv, w.d), "bf16")
    Vp = synth.normal(w.seed, synth.tag(synth.VLOC, layer), (B, L0, w.h_kv, w.d), "bf16")
    n_mem = w.k * 8
    Kb = synth.normal(w.seed, synth.tag(synth.KBAR, layer), (n_mem, w.h_kv, w.d), "bf16")
    Vb = synth.normal(w.seed, synth.tag(synth.VBAR, layer), (n_mem, w.h_kv, w.d), "bf16")
    gi = np.tile(np.arange(n_mem, dtype=np.int32), (B, 1))
    cl = np.full(B, n_mem, np.int32)
    Qs = [synth.normal(w.seed, synth.tag(synth.GEN_Q, layer, s), (B, 1, w.h_q, w.d), "bf16") for s in range(steps)]
    Ks = [synth.normal(w.seed, synth.tag(synth.GEN_K, layer, s), (B, 1, w.h_kv, w.d), "bf16")
          for s in range(steps)]
    Vs = [synth.normal(w.seed, synth.tag(synth.GEN_V, layer, s), (B, 1, w.h_kv, w.d), "bf16")
          for s in range(steps)]
    t0 = time.perf_counter()
    oracle.generate(Qs, Ks, Vs, Kp, Vp, Kb, Vb, gi, cl, w.k, w.rope_base)
    return time.perf_counter() - t0


def cpu_generate_baseline(w, G: int, n_layers: int) -> dict:
    import oracle
    steps = 8
    per_step = statistics.mean(oracle_generate_time(w, l, steps) / steps for l in range(n_layers))
    token = per_step * w.layers
    return {"value": round(w.B / token, 3), "unit": "generated tokens/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"{steps} generation steps of {n_layers} of {w.layers} routed layers "
                       f"(batch {w.B}, 128 memory rows, cache from {w.L_loc} rows); token time = "
                       f"mean step time x {w.layers}; the construction (routing) is left out, so "
                       "this overstates the CPU rate")}


def run_encode_hidden(args):
    """The offline encode from hidden states (msa_encode_hidden) at the 1M-token bank."""
    import torch

    import long_context_doc_b200 as msa
    import synth
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    rank, world = ranks.rank, ranks.world
    w = synth.C2.scaled(seed=synth.C2.seed + 1000 * rank)
    if args.docs > 0:
        w = w.scaled(n_docs=args.docs)
    D, bf = 2560, torch.bfloat16
    off = np.arange(w.n_docs + 1, dtype=np.int64) * w.doc_len
    n_tok = int(off[-1])
    H = synth.dev_normal(torch.empty((n_tok, D), dtype=bf, device=dev), w.seed, synth.tag(50))
    Ws = [synth.dev_normal(torch.empty((w.h_kv * w.d, D), dtype=bf, device=dev), w.seed,
                           synth.tag(51 + i), scale=D ** -0.5) for i in range(3)]
    n_chunks = msa.msa_count_chunks(off, w.chunk)
    shape = (n_chunks, w.h_kv, w.d)
    outs = [torch.empty(shape, dtype=bf, device=dev) for _ in range(3)]
    coff = torch.empty(len(off), dtype=torch.int64, device=dev)
    ws = torch.empty(msa.msa_encode_hidden_workspace(n_chunks), dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream()

    def call():
        msa.msa_encode_hidden(H, *Ws, off, w.chunk, w.rope_base, *outs, coff, ws, st)

    for _ in range(max(args.warmup, 3)):
        call()
    ranks.barrier()
    torch.cuda.synchronize()
    Kst = max(1, min(args.steps, 20))
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(Kst):
        call()
    e1.record(st)
    st.synchronize()
    clocks = sampler.stop()
    assert msa.msa_workspace_status(ws, st) == 0
    # end to end: the hidden states copied from pinned host memory and the pooled bank read
    # back, every call
    host_H = H.cpu().pin_memory()
    host_out = [o.cpu().pin_memory() for o in outs]
    h2d = host_H.numel() * host_H.element_size()
    d2h = sum(o.numel() * o.element_size() for o in host_out)

    def e2e_call():
        with torch.cuda.stream(st):
            H.copy_(host_H, non_blocking=True)
        call()
        with torch.cuda.stream(st):
            for o, ho in zip(outs, host_out):
                ho.copy_(o, non_blocking=True)

    e2e_call()
    st.synchronize()
    Ke = max(1, min(Kst, 3))
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(st)
    for _ in range(Ke):
        e2e_call()
    e3.record(st)
    st.synchronize()
    ms, e2e_ms = ranks.max([e0.elapsed_time(e1) / Kst, e2.elapsed_time(e3) / Ke], dev)
    flop = 2.0 * n_tok * D * 3 * w.h_kv * w.d
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tpeak, tkind = float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        tpeak, tkind = 1400.0, "fallback (sustained)"
    tf = flop / (ms / 1e3) / 1e12
    line = {"metric": "offline encode from hidden states, bank tokens/s (projections + doc-wise "
                      "RoPE + chunk pooling)",
            "value": round(replica_rate(world, n_tok, ms), 1), "unit": "bank tokens/s",
            "n_gpus": world, "steps": Kst, "warmup": max(args.warmup, 3),
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded normals; random "
                                                          "projection weights)",
            "config": {"workload": ("encode_hidden1m" if w.n_docs == 1024 else
                                    f"encode_hidden_{w.n_docs}docs"),
                       "bank_tokens": n_tok, "n_docs": w.n_docs,
                       "hidden": D, "h_kv": w.h_kv, "d": w.d, "chunk": w.chunk,
                       "l2": f"no flush: {n_tok * D * 2 / 1e9:.1f} GB of hidden states per call"},
            "roofline": {"kernel": "encode_hidden_kernel (tcgen05 projections + RoPE + pooling; "
                                   "the call also uploads the chunk table)",
                         "bound": "tensor", "achieved": round(tf, 1), "peak": tpeak,
                         "unit": "TFLOP/s", "frac": round(tf / tpeak, 4), "peak_kind": tkind,
                         "traffic": None},
            "e2e": {"value": round(replica_rate(world, n_tok, e2e_ms), 1), "unit": "bank tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 3)},
            "gpu_launches": Kst, "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_encode_hidden_baseline(w, D)
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def cpu_encode_hidden_baseline(w, D: int, n_docs: int = 8) -> dict:
    """The oracle's encode from hidden states on a sample of the same workload: ``n_docs``
    documents of the bank (their hidden rows, the three projections, RoPE, pooling)."""
    import oracle
    import synth
    off = np.arange(n_docs + 1, dtype=np.int64) * w.doc_len
    n = int(off[-1])
    H = synth.normal(w.seed, synth.tag(50), (n, D), "bf16")
    Wt = [np.ascontiguousarray(synth.normal(w.seed, synth.tag(51 + i), (w.h_kv * w.d, D), "bf16",
                                            scale=D ** -0.5).T) for i in range(3)]
    t0 = time.perf_counter()
    oracle.encode_hidden(H, Wt[0], Wt[1], Wt[2], off, w.chunk, w.rope_base, w.h_kv)
    dt = time.perf_counter() - t0
    return {"value": round(n / dt, 1), "unit": "bank tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{n_docs} of {w.n_docs} documents ({n} tokens), "
                                        "projections + RoPE + pooling"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefill1m":
        run_prefill(args)
    elif args.workload == "interleave10m":
        run_interleave(args)
    elif args.workload == "attend_long":
        run_attend_long(args)
    elif args.workload == "gen100m":
        run_generate(args)
    elif args.workload == "encode_hidden1m":
        run_encode_hidden(args)
    elif args.workload == "attend_bwd":
        run_attend_backward(args)
    elif args.workload == "aux_loss":
        run_aux_loss(args)
    elif args.workload == "fetch100m":
        run_fetch(args)
    else:
        run_libmsa(args)


if __name__ == "__main__":
    main()
