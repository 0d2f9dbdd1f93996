#!/usr/bin/env python
"""Benchmark of the context-sparse decode hot path on B200.

Metric: sparse decode us/step and effective HBM GB/s at 50x sparsity vs dense
decode ("Inference Time Context Sparsity: Illusion or Opportunity?",
gist.science summary, section 3.C: sparse decode kernels against dense decode,
traffic O(k d) instead of O(N d)).

One step runs the whole path on one batch of the workload:
  exact top-k indexer (score + select) -> sparse decode on the selected rows
  -> dense decode on the same cache (the comparator),
each leg captured once into a CUDA graph and replayed between two CUDA events on
the launching stream, with a 256 MiB write and a 256 MiB read (twice the 126 MB
L2) before each leg so every leg reads from HBM.
`value` is the sparse-decode leg (the metric); the other legs are reported
beside it.  Multi-GPU runs are weak scaling: every rank decodes its own batch
(no data-path collective), the timings are the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference] [--config NAME]
                  [--also NAME,NAME]

The default workload is the ragged batch (32 sequences of 8K-128K tokens, 4 decode queries
each, k = ceil(0.02 kv_len)): the largest that fits one GPU.  The three legs of the
Llama-3-8B- and Qwen2.5-72B-shaped workloads are timed too and reported beside it.
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse decode µs/step and effective HBM GB/s at 50× sparsity vs dense decode"
UNIT = "µs/step"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--config", default="ragged",
                   help="workload of the line (default: the ragged batch, the largest single-GPU one)")
    p.add_argument("--also", default="llama3_8b,qwen25_72b",
                   help="comma-separated workloads whose three legs are timed too and reported under "
                        "other_workloads ('' for none)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--record-traffic", metavar="NCU_CSV",
                   help="write profiles/dram_traffic.json for --config from an ncu --csv log of "
                        "dram__bytes_read.sum, dram__bytes_write.sum and gpu__time_duration.sum (no GPU work)")
    p.add_argument("--plain-line", metavar="JSON",
                   help="with --record-traffic: the bench line of the same command run without ncu; its "
                        "sparse-decode algorithmic bytes are stored beside the captured traffic, so that the "
                        "figure can be scaled to a larger copy of the workload")
    p.add_argument("--traffic-command", metavar="CMD",
                   help="with --record-traffic: the ncu command that made the log, stored with the figure")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_desc(cfg, k):
    return {
        "workload": f"{cfg.name}: {cfg.description}",
        "batch": cfg.batch, "q_heads": cfg.num_q_heads, "kv_heads": cfg.num_kv_heads, "head_dim": 128,
        "context": cfg.max_seq_len, "k": k, "tokens_per_seq": cfg.tokens_per_seq,
        "l2": "flushed before every timed leg: 256 MiB device write, then a 256 MiB read (no input, and "
              "none of the flush's dirty lines, left in L2)",
        "timing": "each leg (its library call) captured once into a CUDA graph; CUDA events around every "
                  "replay on the launching stream",
    }


class L2Flush:
    """Evict L2 (126 MB on B200) before a timed leg: write a 256 MiB buffer, then read another
    256 MiB one.  The read pushes the write's dirty lines out of L2 too, so the timed kernel
    neither finds its inputs in L2 nor pays for writing back lines the flush left dirty."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(32 << 20, dtype=torch.int64, device=dev)
        self.sink = torch.zeros((), dtype=torch.int64, device=dev)

    def __call__(self):
        import torch
        self.w.fill_(1)
        torch.sum(self.r, dim=0, out=self.sink)


# ---------------------------------------------------------------------------
# Clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for r in csv.reader(io.StringIO(self.out or "")):
            if len(r) < 9:
                continue
            try:
                rows.append([x.strip() for x in r])
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = sorted(float(r[1]) for r in rows if r[1].replace('.', '', 1).isdigit())
        smax = max((float(r[2]) for r in rows if r[2].replace('.', '', 1).isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j].lower().startswith("active")})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# Helpers
# ---------------------------------------------------------------------------
# files whose contents decide the sparse kernel and its launch shape
SPARSE_SOURCES = ["tsd_decode.cu", "tsd_plan.h", "tsd_common.cuh"]


def source_sha(names):
    """Hash of the kernel sources (file names under csrc/, or one name), in order."""
    if isinstance(names, str):
        names = [names]
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "top_sparse_decode_topk_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# workloads whose traffic is captured on a reduced copy (the full size is beyond a detailed
# profiler capture): the copy's DRAM bytes per algorithmic byte, times the full launch's
# algorithmic bytes
TRAFFIC_SCALED_FROM = {"ragged": "ragged_8", "qwen25_72b": "qwen25_72b_b2"}


def ncu_traffic(kernel: str, workload: str, source, algorithmic_bytes=None):
    """(DRAM bytes per launch, how) from the committed ncu summary, if it was taken on the
    current kernel source (else (None, reason)).  A workload captured only as a reduced copy
    gets the copy's DRAM/algorithmic ratio times its own algorithmic bytes."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None, "no capture recorded"
    rec = d.get(kernel, {})
    for name, scaled in ((workload, False), (TRAFFIC_SCALED_FROM.get(workload), True)):
        e = rec.get(name) if name else None
        if e is None:
            continue
        if e.get("source_sha") != source_sha(source):
            return None, f"the {name} capture predates the current kernel source"
        if not scaled:
            return float(e["bytes_per_launch"]), f"ncu capture of {name}"
        if algorithmic_bytes is None or not e.get("algorithmic_bytes"):
            return None, f"the {name} capture has no algorithmic bytes to scale by"
        ratio = float(e["bytes_per_launch"]) / float(e["algorithmic_bytes"])
        return ratio * algorithmic_bytes, (f"ncu capture of {name} (DRAM/algorithmic = {ratio:.4f}), scaled "
                                           f"to this launch's algorithmic bytes")
    return None, "no capture of this kernel on this workload"


# kernel -> the csrc files that decide its code and launch shape
KERNEL_SOURCES = {
    "sparse_decode_kernel": SPARSE_SOURCES,
    "sparse_stream_kernel": SPARSE_SOURCES,
    "dense_decode_kernel": ["tsd_decode.cu", "tsd_plan.h", "tsd_common.cuh", "tsd_kvtile.cuh"],
    "topk_score_kernel": ["tsd_topk.cu", "tsd_plan.h", "tsd_common.cuh", "tsd_kvtile.cuh"],
    "topk_select_kernel": ["tsd_topk.cu", "tsd_plan.h", "tsd_common.cuh"],
}


def record_traffic(csv_path: str, workload: str, plain_line: str = None, command: str = None):
    """Fold one ncu --csv metric log into profiles/dram_traffic.json (first launch of each kernel)."""
    alg = None
    if plain_line:
        with open(plain_line) as f:
            alg = json.loads(f.read().strip().splitlines()[-1])["roofline"]["algorithmic_bytes"]
    import csv
    with open(csv_path) as f:
        rows = list(csv.reader(f))
    head = [i for i, r in enumerate(rows) if r and r[0] == "ID"][0]
    h = rows[head]
    got = {}
    for r in rows[head + 1:]:
        d = dict(zip(h, r))
        name = d.get("Kernel Name", "")
        kern = next((k for k in KERNEL_SOURCES if k in name), None)
        if kern is None:
            continue
        e = got.setdefault(kern, {"id": d["ID"]})
        if e["id"] != d["ID"]:
            continue   # a later launch of the same kernel
        e[d["Metric Name"]] = float(d["Metric Value"].replace(",", ""))
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            out = json.load(f)
    except Exception:
        out = {}
    out.setdefault("_about", "DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of one captured "
                   "launch per kernel and workload, L2 flushed before it (the bench's own flush); bench.py uses a "
                   "kernel's figure as roofline.traffic only while source_sha still matches the kernel's sources. "
                   "Each entry gives the command that made it.")
    for kern, e in got.items():
        rd, wr = e.get("dram__bytes_read.sum"), e.get("dram__bytes_write.sum")
        if rd is None or wr is None:
            continue
        out.setdefault(kern, {})[workload] = {
            "bytes_per_launch": rd + wr, "read": rd, "write": wr,
            "duration_us": round(e.get("gpu__time_duration.sum", float("nan")) / 1e3, 3),
            "sources": KERNEL_SOURCES[kern], "source_sha": source_sha(KERNEL_SOURCES[kern])}
        if command:
            out[kern][workload]["command"] = command
        if alg is not None and kern.startswith("sparse_"):
            out[kern][workload]["algorithmic_bytes"] = alg
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps({k: v for k, v in out.items() if k != "_about"}, indent=1))



def unique_rows(idx, token_seq, hkv, group, max_len):
    """Distinct (sequence, kv head, token) rows named by the index lists."""
    import torch
    T, Hq, K = idx.shape
    b = token_seq.view(T, 1, 1).long()
    g = (torch.arange(Hq, device=idx.device) // group).view(1, Hq, 1)
    key = (b * hkv + g) * max_len + idx.long()
    key = key[idx >= 0]
    return int(torch.unique(key).numel())


def _oracle_sparse_worker(payload):
    """One process of the all-cores oracle timing: attach to the group's K and V (shared
    memory), then repeat the oracle's sparse attention of one list for `budget_s`; return
    (evaluations, seconds)."""
    from multiprocessing import shared_memory
    import numpy as np
    q, kname, vname, shape, L, ix, scale, budget_s = payload
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    import oracle
    ks, vs = shared_memory.SharedMemory(name=kname), shared_memory.SharedMemory(name=vname)
    try:
        K = np.ndarray(shape, dtype=np.float64, buffer=ks.buf)[:L]
        V = np.ndarray(shape, dtype=np.float64, buffer=vs.buf)[:L]
        t0 = time.perf_counter()
        n = 0
        while True:
            oracle.sparse_attention(q, K, V, ix, scale)
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        el = time.perf_counter() - t0
        del K, V
    finally:
        ks.close()
        vs.close()
    return n, el


def time_cpu_oracle_all_cores(groups_kv, lists, total_lists, scale, budget_s=5.0):
    """The oracle's sparse attention on every usable host core at once: one spawned process per
    core, each repeating one sampled list against its group's full K and V (shared memory, not
    copied) for `budget_s`.  List evaluations per second over all processes, as µs per step."""
    import multiprocessing as mp
    from multiprocessing import shared_memory
    import numpy as np
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    shms = []
    try:
        names = []
        for K, V in groups_kv:
            pair = []
            for A in (K, V):
                sm = shared_memory.SharedMemory(create=True, size=A.nbytes)
                shms.append(sm)
                np.ndarray(A.shape, dtype=np.float64, buffer=sm.buf)[:] = A
                pair.append(sm.name)
            names.append((pair[0], pair[1], K.shape))
        payloads = []
        for i in range(cores):
            q, gi, L, ix = lists[i % len(lists)]
            kname, vname, shape = names[gi]
            payloads.append((q, kname, vname, shape, L, ix, scale, budget_s))
        with mp.get_context("spawn").Pool(cores) as pool:   # bounded wait: a failed worker raises here
            res = pool.map_async(_oracle_sparse_worker, payloads).get(timeout=4 * budget_s + 120)
    finally:
        for sm in shms:
            sm.close()
            sm.unlink()
    rate = sum(n for n, _ in res) / max(s for _, s in res)   # list evaluations per second
    return {"value": total_lists / rate * 1e6, "cores": cores,
            "sample": f"{len(lists)} sampled lists spread over {cores} spawned processes (one per core), "
                      f"~{budget_s:.0f} s each, lists per second scaled to the full step"}


def time_cpu_oracle(w, k, budget_s=10.0):
    """The oracle on the host cores: exact top-k plus sparse attention for a sample of
    (sequence, kv head) groups, repeated until `budget_s`; extrapolated to the step."""
    import numpy as np
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1)
    except Exception:
        limiter = None
    import oracle
    cfg = w.cfg
    G = cfg.group
    scale = 1.0 / math.sqrt(128)
    rng = np.random.default_rng(0)
    groups = [(int(rng.integers(cfg.batch)), int(rng.integers(cfg.num_kv_heads))) for _ in range(2)]
    data = []
    groups_kv, where, toks = [], [], []
    for b, g in groups:
        K = oracle.from_bf16_bits(w.logical_kv_bits(b, g, "k"))
        V = oracle.from_bf16_bits(w.logical_kv_bits(b, g, "v"))
        groups_kv.append((K, V))
        for t in range(int(w.q_indptr[b]), int(w.q_indptr[b + 1])):
            L = int(w.kv_len[t])
            for h in range(g * G, (g + 1) * G):
                data.append((oracle.from_bf16_bits(w.q_bits[t, h]), K[:L], V[:L]))
                where.append((len(groups_kv) - 1, L))
                toks.append(t)
    nlists = len(data)
    total_lists = len(w.kv_len) * cfg.num_q_heads
    kk = w.k_per_token(k)
    idxs = [oracle.exact_topk(oracle.attention_scores(q, Kb), int(kk[t])) for (q, Kb, _), t in zip(data, toks)]
    # top-k
    t0 = time.perf_counter()
    reps_topk = 0
    while True:
        for (q, Kb, _), t in zip(data, toks):
            oracle.exact_topk(oracle.attention_scores(q, Kb), int(kk[t]))
        reps_topk += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    topk_s = (time.perf_counter() - t0) / reps_topk
    # sparse attention over the selected lists
    t0 = time.perf_counter()
    reps = 0
    while True:
        for (q, Kb, Vb), ix in zip(data, idxs):
            oracle.sparse_attention(q, Kb, Vb, ix, scale)
        reps += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    sparse_s = (time.perf_counter() - t0) / reps
    f = total_lists / nlists
    try:
        all_cores = time_cpu_oracle_all_cores(
            groups_kv, [(q, gi, L, ix) for (q, _, _), (gi, L), ix in zip(data, where, idxs)], total_lists, scale)
    except Exception as e:   # a host that cannot spawn workers still reports the one-core figure
        all_cores = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    return {
        "sparse_us_per_step": sparse_s * f * 1e6,
        "topk_us_per_step": topk_s * f * 1e6,
        "all_cores": all_cores,
        "cores": 1,
        "sample": f"{nlists} of {total_lists} (token, head) lists ({len(groups)} (sequence, kv head) groups), "
                  f"{reps} repetitions of the sparse attention and {reps_topk} of the top-k in "
                  f"~{budget_s:.0f} s, extrapolated linearly to the full step",
    }


# ---------------------------------------------------------------------------
# Native arm
# ---------------------------------------------------------------------------
def bench_k(cfg):
    """k of the bench line: the configuration's k nearest the 50x sparsity the metric names
    (None: the configuration's own per-token rule, ceil(frac * kv_len))."""
    if not cfg.ks:
        return None
    target = cfg.max_seq_len / 50.0
    return min(cfg.ks, key=lambda k: abs(k - target))


def rank_seed(rank: int) -> int:
    """Seed of a rank's workload: every rank decodes its own batch of sequences (weak scaling)."""
    return rank


def max_over_ranks(values, device):
    """Element-wise MAX of per-rank timings over the process group (identity on one process).
    Every rank must call it with the same number of values, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device):
    """Element-wise SUM over the process group (identity on one process)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def leg_graph(fn):
    """`fn` (one leg: its library calls, buffers already sized by an eager run) captured once
    into a CUDA graph.  The timed region then replays it: the whole leg is enqueued in one call,
    so host-side launch overhead never leaves the GPU idle inside the events."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_legs(tsd, W, name, rank, dev, steps, warmup, flush):
    """The three legs (exact top-k, sparse decode at the workload's 50x k, dense decode) of one more
    workload, timed like the line's own legs (CUDA events, L2 flushed before each), with the
    algorithmic bytes of each.  Every rank runs it on its own batch; the caller reduces."""
    import numpy as np
    import torch
    cfg = W.CONFIGS[name]
    k = bench_k(cfg)
    w = W.make_workload(cfg, seed=rank_seed(rank))
    dw = W.to_device(w, dev)
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=cfg.max_seq_len,
                        page_table=None if cfg.layout == "contiguous" else dw.page_table)
    multi = cfg.tokens_per_seq > 1
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                          causal=cfg.causal, sm_scale=1.0 / math.sqrt(128))
    kpt = w.k_per_token(k)
    k_max = int(kpt.max())
    kpt_dev = None if k is not None else torch.from_numpy(kpt).to(dev)
    odt = torch.float32 if cfg.out_dtype == "f32" else torch.bfloat16
    ws = tsd.Workspace(dev)
    stream = torch.cuda.current_stream(dev)
    T, Hq = len(w.kv_len), cfg.num_q_heads
    idx = torch.empty((T, Hq, k_max), dtype=torch.int32, device=dev)
    cnt = torch.empty((T, Hq), dtype=torch.int32, device=dev)
    legs = [lambda: tsd.topk_select(cache, queries, k_max, k_per_token=kpt_dev, out_idx=idx, out_count=cnt,
                                    workspace=ws),
            lambda: tsd.sparse_decode(cache, queries, idx, out_dtype=odt, workspace=ws),
            lambda: tsd.dense_decode(cache, queries, out_dtype=odt, workspace=ws)]
    for _ in range(max(3, warmup)):
        for leg in legs:
            flush()
            leg()
    graphs = [leg_graph(leg) for leg in legs]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    torch.cuda.synchronize()
    for s_ in range(steps):
        for j, g in enumerate(graphs):
            flush()
            ev[s_][2 * j].record(stream)
            g.replay()
            ev[s_][2 * j + 1].record(stream)
    torch.cuda.synchronize()
    del graphs
    if tsd.read_device_status(ws) != 0:
        raise RuntimeError(f"device status bits set on {name}")
    ms = np.array([[ev[s_][2 * j].elapsed_time(ev[s_][2 * j + 1]) for j in range(3)] for s_ in range(steps)])
    U = unique_rows(idx, torch.from_numpy(w.token_seq).to(dev), cfg.num_kv_heads, cfg.group, cfg.max_seq_len)
    ob = 4 if odt == torch.float32 else 2
    q_bytes, o_bytes = T * Hq * 128 * 2, T * Hq * 128 * ob
    ctx_rows = int(sum(int(L) for L in w.seq_lens)) * cfg.num_kv_heads
    nbytes = [ctx_rows * 256 + q_bytes + T * Hq * k_max * 4, U * 512 + q_bytes + o_bytes,
              ctx_rows * 512 + q_bytes + o_bytes]
    del cache, queries, dw, ws, idx, cnt
    torch.cuda.empty_cache()
    return ms.mean(axis=0).tolist(), nbytes, k_max, U


def run_native(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import top_sparse_decode_topk_b200 as tsd
    from top_sparse_decode_topk_b200 import workload as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from top_sparse_decode_topk_b200.build import build
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    tsd.load_library()

    cfg = W.CONFIGS[args.config]
    k = bench_k(cfg)
    w = W.make_workload(cfg, seed=rank_seed(rank))
    dw = W.to_device(w, dev)
    contiguous = cfg.layout == "contiguous"
    cache = tsd.KVCache(dw.k, dw.v, dw.seq_lens, max_seq_len=cfg.max_seq_len,
                        page_table=None if contiguous else dw.page_table)
    multi = cfg.tokens_per_seq > 1
    scale = 1.0 / math.sqrt(128)
    queries = tsd.Queries(dw.q, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                          causal=cfg.causal, sm_scale=scale)
    kpt = w.k_per_token(k)
    k_max = int(kpt.max())
    kpt_dev = None if k is not None else torch.from_numpy(kpt).to(dev)
    out_dtype = torch.float32 if cfg.out_dtype == "f32" else torch.bfloat16
    ws = tsd.Workspace(dev)
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)
    idx_buf = torch.empty((len(w.kv_len), cfg.num_q_heads, k_max), dtype=torch.int32, device=dev)
    cnt_buf = torch.empty((len(w.kv_len), cfg.num_q_heads), dtype=torch.int32, device=dev)

    def leg_topk():
        tsd.topk_select(cache, queries, k_max, k_per_token=kpt_dev, out_idx=idx_buf, out_count=cnt_buf, workspace=ws)

    def leg_sparse():
        return tsd.sparse_decode(cache, queries, idx_buf, out_dtype=out_dtype, workspace=ws)

    def leg_dense():
        return tsd.dense_decode(cache, queries, out_dtype=out_dtype, workspace=ws)

    legs = [leg_topk, leg_sparse, leg_dense]
    for _ in range(max(3, args.warmup)):
        for leg in legs:
            flush()
            leg()
    torch.cuda.synchronize()
    if tsd.read_device_status(ws) != 0:
        raise RuntimeError("device status bits set during warm-up")
    leg_graphs = [leg_graph(leg) for leg in legs]

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for s in range(args.steps):
            for j, g in enumerate(leg_graphs):
                flush()
                ev[s][2 * j].record(stream)
                g.replay()
                ev[s][2 * j + 1].record(stream)
        torch.cuda.synchronize()
    del leg_graphs
    if world > 1:
        dist.barrier()
    ms = np.array([[ev[s][2 * j].elapsed_time(ev[s][2 * j + 1]) for j in range(3)] for s in range(args.steps)])
    mean_ms = ms.mean(axis=0)
    topk_ms, sparse_ms, dense_ms = max_over_ranks(mean_ms.tolist(), dev)

    # algorithmic bytes (per rank; every rank has the same shapes)
    T, Hq, Hkv, G = len(w.kv_len), cfg.num_q_heads, cfg.num_kv_heads, cfg.group
    U = unique_rows(idx_buf, torch.from_numpy(w.token_seq).to(dev), Hkv, G, cfg.max_seq_len)
    entries = int((idx_buf >= 0).sum().item())
    out_bytes = 4 if out_dtype == torch.float32 else 2
    q_bytes = T * Hq * 128 * 2
    o_bytes = T * Hq * 128 * out_bytes
    sparse_bytes = U * 512 + q_bytes + o_bytes
    ctx_rows = int(sum(int(L) for L in w.seq_lens)) * Hkv
    dense_bytes = ctx_rows * 512 + q_bytes + o_bytes
    topk_bytes = ctx_rows * 256 + q_bytes + T * Hq * k_max * 4
    index_bytes = T * Hq * k_max * 4
    hbm, peak_kind = peaks()
    topk_plan = tsd.topk_select_plan(cache, queries, k_max)
    topk_form = ("candidate-filtered: sample pre-pass, per-list thresholds, scoring that keeps only the "
                 "scores reaching them, selection among those" if topk_plan["filtered"]
                 else "full score rows, then selection over each row")
    # whole-job bytes (each rank decodes its own batch) over the slowest rank's time; the
    # roofline is per GPU: the job's bytes per GPU over that time
    job_sparse, job_dense, job_topk = sum_over_ranks([sparse_bytes, dense_bytes, topk_bytes], dev)
    gbs = lambda b, ms_: b / (ms_ * 1e-3) / 1e9
    job_sparse_gbs = gbs(job_sparse, sparse_ms)
    sparse_gbs, dense_gbs, topk_gbs = (gbs(job_sparse / world, sparse_ms), gbs(job_dense / world, dense_ms),
                                       gbs(job_topk / world, topk_ms))

    # label-channel (Double-Sparsity-style) indexer: offline calibration once, then the
    # decode-step cost of approximate top-k + sparse decode against dense decode over a
    # sparsity sweep, next to the exact indexer's
    def timed(fn, reps):
        out = []
        for _ in range(reps):
            flush()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            fn()
            b_.record(stream)
            torch.cuda.synchronize()
            out.append(a_.elapsed_time(b_))
        return float(np.mean(out[1:])) if len(out) > 1 else out[0]

    r_label = 16
    t_cal = timed(lambda: tsd.label_channels(cache, queries, r_label), 2)
    channels = tsd.label_channels(cache, queries, r_label)
    label_index = tsd.label_cache_build(cache, channels)
    torch.cuda.synchronize()
    curve = []
    reps = max(4, args.steps // 4 + 1)
    for x in (2, 5, 10, 20, 50, 100, 200):
        kx = W.k_for_sparsity(cfg.max_seq_len, x)
        ibuf = torch.empty((T, Hq, kx), dtype=torch.int32, device=dev)
        cbuf = torch.empty((T, Hq), dtype=torch.int32, device=dev)
        t_lab = timed(lambda: tsd.topk_select_label(cache, label_index, queries, kx, out_idx=ibuf, out_count=cbuf,
                                                    workspace=ws), reps)
        t_ex = timed(lambda: tsd.topk_select(cache, queries, kx, out_idx=ibuf, out_count=cbuf, workspace=ws), reps)
        t_sp = timed(lambda: tsd.sparse_decode(cache, queries, ibuf, out_dtype=out_dtype, workspace=ws), reps)
        t_lab, t_ex, t_sp = max_over_ranks([t_lab, t_ex, t_sp], dev)
        curve.append({"sparsity": x, "k": kx, "label_topk_us": round(t_lab * 1e3, 2),
                      "exact_topk_us": round(t_ex * 1e3, 2), "sparse_us": round(t_sp * 1e3, 2),
                      "net_speedup_label": round(dense_ms / (t_lab + t_sp), 3),
                      "net_speedup_exact": round(dense_ms / (t_ex + t_sp), 3)})
    if tsd.read_device_status(ws) != 0:
        raise RuntimeError("device status bits set in the label-indexer sweep")
    label_line = {"r": r_label, "calibration_us": round(max_over_ranks([t_cal], dev)[0] * 1e3, 1),
                  "label_cache_bytes": int(label_index.label_k.numel() * 2),
                  "dense_us": round(dense_ms * 1e3, 3), "curve": curve,
                  "what": "label top-k (r channels per kv head, exact top-k of the approximate scores) and "
                          "exact top-k, each plus sparse decode, against dense decode on the same cache"}

    # the decode step on the device as one CUDA graph: indexer (exact, or label channels) then
    # sparse decode on the same workspace, replayed with L2 flushed before each replay; and the
    # sparse leg alone as a graph (what its launch costs outside a graph)
    out_g = torch.empty((T, Hq, 128), dtype=out_dtype, device=dev)
    lse_g = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    kpt_g = kpt_dev

    def step_exact():   # the library's one-call step (tsd_decode_step)
        tsd.decode_step(cache, queries, k_max, k_per_token=kpt_g, out_idx=idx_buf, out_count=cnt_buf, out=out_g,
                        lse=lse_g, workspace=ws)

    def step_label():
        tsd.topk_select_label(cache, label_index, queries, k_max, k_per_token=kpt_g, out_idx=idx_buf,
                              out_count=cnt_buf, workspace=ws)
        tsd.sparse_decode(cache, queries, idx_buf, out=out_g, lse=lse_g, workspace=ws)

    def sparse_only():
        tsd.sparse_decode(cache, queries, idx_buf, out=out_g, lse=lse_g, workspace=ws)

    # vAttention-style: exact top-k plus m uniform samples of the rest, weighted decode
    m_sto = 64
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    u_sto = torch.randint(-2**31, 2**31 - 1, (T, Hq, m_sto), dtype=torch.int32, device=dev, generator=gen)

    def step_stochastic():
        tsd.topk_select(cache, queries, k_max, k_per_token=kpt_g, out_idx=idx_buf, out_count=cnt_buf, workspace=ws)
        sidx, slw = tsd.stochastic_select(cache, queries, idx_buf, u_sto)
        tsd.sparse_decode(cache, queries, sidx, logw=slw, out=out_g, lse=lse_g, workspace=ws)

    graph_us = {}
    for name, fn in (("sparse_decode", sparse_only), ("step_exact_indexer", step_exact),
                     ("step_label_indexer", step_label), ("step_stochastic", step_stochastic)):
        fn()   # warm: buffers exist, launch attributes set
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        graph_us[name] = timed(g.replay, reps + 1)
        del g
    torch.cuda.synchronize()
    if tsd.read_device_status(ws) != 0:
        raise RuntimeError("device status bits set in the graph-captured steps")
    gx = max_over_ranks([graph_us["sparse_decode"], graph_us["step_exact_indexer"], graph_us["step_label_indexer"],
                         graph_us["step_stochastic"]], dev)
    graph_line = {"sparse_decode_us": round(gx[0] * 1e3, 2), "step_exact_indexer_us": round(gx[1] * 1e3, 2),
                  "step_label_indexer_us": round(gx[2] * 1e3, 2),
                  "step_stochastic_us": round(gx[3] * 1e3, 2), "stochastic_samples": m_sto,
                  "net_speedup_exact": round(dense_ms / gx[1], 3), "net_speedup_label": round(dense_ms / gx[2], 3),
                  "net_speedup_stochastic": round(dense_ms / gx[3], 3),
                  "what": "one CUDA graph per decode step (indexer + sparse decode, k of this line; the exact "
                          "step is one tsd_decode_step call; the "
                          "stochastic step adds m uniform samples of the other tokens with Horvitz-Thompson "
                          "weights and decodes with them), L2 flushed before each replay; dense decode by "
                          "events as in legs_us"}

    # A second figure: 20 sparse-decode steps back to back in one CUDA graph, each over its own
    # index set (the top-k lists of a different seeded random query batch), L2 flushed once before
    # each replay.  Launches are pipelined here, so this is the per-step time without the
    # launch-and-event overhead of a single timed call.
    n_rot = 20
    gq = torch.Generator(device=dev)
    gq.manual_seed(4321 + rank)
    rot = []
    rot_bytes = 0
    for _ in range(n_rot):
        qi = torch.randn(dw.q.shape, device=dev, generator=gq).to(dw.q.dtype)
        qsi = tsd.Queries(qi, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                          causal=cfg.causal, sm_scale=scale)
        ii = torch.empty_like(idx_buf)
        tsd.topk_select(cache, qsi, k_max, k_per_token=kpt_dev, out_idx=ii, out_count=torch.empty_like(cnt_buf),
                        workspace=ws)
        rot.append((qsi, ii))
        rot_bytes += unique_rows(ii, torch.from_numpy(w.token_seq).to(dev), Hkv, G, cfg.max_seq_len) * 512
    rot_bytes += n_rot * (q_bytes + o_bytes)

    def rot_steps():
        for qsi, ii in rot:
            tsd.sparse_decode(cache, qsi, ii, out=out_g, lse=lse_g, workspace=ws)

    rot_steps()
    torch.cuda.synchronize()
    g20 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g20):
        rot_steps()
    t20 = timed(g20.replay, reps + 1)
    del g20
    torch.cuda.synchronize()
    if tsd.read_device_status(ws) != 0:
        raise RuntimeError("device status bits set in the rotating-index graph")
    t20 = max_over_ranks([t20], dev)[0]
    rot_us = t20 * 1e3 / n_rot
    rot_gbs = gbs(rot_bytes / n_rot, t20 / n_rot)
    graph20_line = {"sparse_decode_us_per_step": round(rot_us, 3), "steps": n_rot,
                    "achieved_gbs": round(rot_gbs, 1), "frac": round(rot_gbs / hbm, 4),
                    "what": "20 sparse-decode steps back to back in one CUDA graph, each over the top-k lists of a "
                            "different seeded random query batch; L2 flushed once before each replay; bytes are "
                            "each step's own unique rows + q + out"}
    sp_samples = ms[:, 1] * 1e3
    sparse_stats = dict(zip(("median", "min", "p90"), max_over_ranks(
        [float(np.median(sp_samples)), float(np.min(sp_samples)), float(np.percentile(sp_samples, 90))], dev)))
    sparse_stats = {k_: round(v_, 3) for k_, v_ in sparse_stats.items()}

    # end to end through the public API with pinned host buffers
    q_host = dw.q.cpu().pin_memory()
    idx_host = idx_buf.cpu().pin_memory()
    out_host = torch.empty((T, Hq, 128), dtype=out_dtype).pin_memory()
    lse_host = torch.empty((T, Hq), dtype=torch.float32).pin_memory()
    hq = tsd.Queries(q_host, q_indptr=dw.q_indptr if multi else None, max_tokens_per_seq=cfg.tokens_per_seq,
                     causal=cfg.causal, sm_scale=scale)
    e2e_ms, e2e_idx_ms = [], []
    for s in range(args.warmup + args.steps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tsd.sparse_decode(cache, hq, idx_host, out=out_host, lse=lse_host, workspace=ws)
        b.record(stream)
        flush()
        c, d = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c.record(stream)
        # q crosses to the device once (inside the timed region) and serves both calls
        qdev = tsd.Queries(hq.q.to(dev, non_blocking=True), q_indptr=hq.q_indptr,
                           max_tokens_per_seq=hq.max_tokens_per_seq, causal=hq.causal, sm_scale=hq.sm_scale)
        idx_d, _ = tsd.topk_select(cache, qdev, k_max, k_per_token=kpt_dev, out_idx=idx_buf, out_count=cnt_buf,
                                   workspace=ws)
        tsd.sparse_decode(cache, qdev, idx_d, out=out_host, lse=lse_host, workspace=ws)
        d.record(stream)
        torch.cuda.synchronize()
        if s >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
            e2e_idx_ms.append(c.elapsed_time(d))
    e2e_us, e2e_idx_us = (x * 1e3 for x in max_over_ranks([np.mean(e2e_ms), np.mean(e2e_idx_ms)], dev))
    if tsd.read_device_status(ws) != 0:
        raise RuntimeError("device status bits set during the timed run")

    # the three legs of the other workloads named by --also (every rank, same order)
    others = {}
    for name in [x for x in args.also.split(",") if x and x != cfg.name]:
        x_ms, x_bytes, x_k, x_u = time_legs(tsd, W, name, rank, dev, max(3, args.steps // 2), args.warmup, flush)
        x_ms = max_over_ranks(x_ms, dev)
        x_gbs = [gbs(b_, m_) for b_, m_ in zip(x_bytes, x_ms)]
        others[name] = {
            "k": x_k, "unique_rows": x_u,
            "legs_us": {"topk_select": round(x_ms[0] * 1e3, 3), "sparse_decode": round(x_ms[1] * 1e3, 3),
                        "dense_decode": round(x_ms[2] * 1e3, 3)},
            "achieved_gbs": {"topk_select": round(x_gbs[0], 1), "sparse_decode": round(x_gbs[1], 1),
                             "dense_decode": round(x_gbs[2], 1)},
            "frac_of_peak": {"topk_select": round(x_gbs[0] / hbm, 4), "sparse_decode": round(x_gbs[1] / hbm, 4),
                             "dense_decode": round(x_gbs[2] / hbm, 4)},
            "speedup_vs_dense": round(x_ms[2] / x_ms[1], 3),
            "speedup_vs_dense_with_indexer": round(x_ms[2] / (x_ms[0] + x_ms[1]), 3),
            "algorithmic_bytes": {"topk_select": x_bytes[0], "sparse_decode": x_bytes[1],
                                  "dense_decode": x_bytes[2]}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_cpu_oracle(w, k)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    cl = clocks.summary()
    plan = tsd.sparse_decode_plan(cache, queries, k_max)
    traffic, traffic_how = ncu_traffic(plan["kernel"], cfg.name, SPARSE_SOURCES, sparse_bytes)
    line = {
        "metric": METRIC,
        "value": round(sparse_ms * 1e3, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(topk_ms + sparse_ms + dense_ms, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "dtype_detail": "bf16 K/V/q storage; q.K and P.V on bf16 tensor-core MMAs (mma.sync m16n8k16) with fp32 "
                        "accumulation; the softmax weights enter P.V as a bf16 hi + lo pair (about 16 significant "
                        "bits); softmax, split merge and normalisation in fp32; "
                        + ("fp32 output" if out_dtype == torch.float32 else "bf16 output"),
        "data": "synthetic (seeded Philox N(0,1) bf16 K/V/q with planted needles/sink/window)"
                if cfg.planted else "synthetic (seeded Philox N(0,1) bf16 K/V/q)",
        "config": workload_desc(cfg, k_max),
        "legs_us": {"topk_select": round(topk_ms * 1e3, 3), "sparse_decode": round(sparse_ms * 1e3, 3),
                    "dense_decode": round(dense_ms * 1e3, 3)},
        "effective_gbs": round(job_sparse_gbs, 1),
        "effective_gbs_per_gpu": round(sparse_gbs, 1),
        "speedup_vs_dense": round(dense_ms / sparse_ms, 3),
        "speedup_vs_dense_with_indexer": round(dense_ms / (sparse_ms + topk_ms), 3),
        "roofline": {"bound": "hbm", "achieved": round(sparse_gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(sparse_gbs / hbm, 4),
                     "traffic": None if traffic is None else round(traffic), "traffic_source": traffic_how,
                     "kernel": plan["kernel"], "plan": plan, "peak_source": f"{peak_kind} copy bandwidth",
                     "frac_of_nominal_8tbs": round(sparse_gbs / NOMINAL_HBM_GBS, 4),
                     "algorithmic_bytes": sparse_bytes, "unique_rows": U, "entries": entries,
                     "index_bytes_not_counted": index_bytes},
        "rooflines_other": {
            "topk_select": {"achieved": round(topk_gbs, 1), "frac": round(topk_gbs / hbm, 4),
                            "algorithmic_bytes": topk_bytes, "form": topk_form,
                            "kernels": (["topk_prepass_kernel", "topk_score_kernel", "topk_cand_kernel",
                                         "topk_select_kernel (queue pass)"] if topk_plan["filtered"]
                                        else ["topk_score_kernel", "topk_select_kernel"])},
            "dense_decode": {"achieved": round(dense_gbs, 1), "frac": round(dense_gbs / hbm, 4),
                             "algorithmic_bytes": dense_bytes, "kernels": ["dense_decode_kernel"]},
        },
        "e2e": {"value": round(e2e_us, 3), "unit": UNIT, "h2d_bytes_per_step": q_bytes + index_bytes,
                "d2h_bytes_per_step": o_bytes + T * Hq * 4,
                "what": "tsd.sparse_decode with pinned host q and index lists in, host out and lse back"},
        "e2e_with_indexer": {"value": round(e2e_idx_us, 3), "unit": UNIT, "h2d_bytes_per_step": q_bytes,
                             "d2h_bytes_per_step": o_bytes + T * Hq * 4,
                             "what": "host q in -> topk_select -> sparse_decode -> host out and lse"},
        "label_indexer": label_line,
        "graph_step": graph_line,
        "graph20_rotating": graph20_line,
        "sparse_leg_us_stats": sparse_stats,
        "other_workloads": others,
        "gpu_launches": (topk_plan["kernels"] + 2) * args.steps,
        "clocks": cl,
    }
    if cpu is not None:
        ac = dict(cpu["all_cores"])
        if "value" in ac:
            ac["value"] = round(ac["value"], 1)
            ac["unit"] = UNIT
        line["cpu_baseline"] = {"value": round(cpu["sparse_us_per_step"], 1), "unit": UNIT, "cores": cpu["cores"],
                                "kind": "oracle", "sample": cpu["sample"],
                                "topk_us_per_step": round(cpu["topk_us_per_step"], 1),
                                "all_cores": ac}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Reference arm: the CPU oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    from top_sparse_decode_topk_b200 import workload as W
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    cfg = W.CONFIGS[args.config]
    k = bench_k(cfg)
    w = W.make_workload(cfg, seed=0)
    G = cfg.group
    scale = 1.0 / math.sqrt(128)
    rng = np.random.default_rng(0)
    groups = [(int(rng.integers(cfg.batch)), int(rng.integers(cfg.num_kv_heads))) for _ in range(2)]
    kk = w.k_per_token(k)
    data = []
    for b, g in groups:
        K = oracle.from_bf16_bits(w.logical_kv_bits(b, g, "k"))
        V = oracle.from_bf16_bits(w.logical_kv_bits(b, g, "v"))
        for t in range(int(w.q_indptr[b]), int(w.q_indptr[b + 1])):
            L = int(w.kv_len[t])
            for h in range(g * G, (g + 1) * G):
                q = oracle.from_bf16_bits(w.q_bits[t, h])
                idx = oracle.exact_topk(oracle.attention_scores(q, K[:L]), int(kk[t]))
                data.append((q, K[:L], V[:L], idx))
    total = len(w.kv_len) * cfg.num_q_heads
    f = total / len(data)
    times = []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for q, Kb, Vb, idx in data:
            oracle.sparse_attention(q, Kb, Vb, idx, scale)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt * f * 1e6)
    v = float(np.mean(times))
    sample = (f"{len(data)} of {total} (token, head) lists ({len(groups)} (sequence, kv head) groups) per step, "
              f"extrapolated linearly to the full step")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v / 1e3, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_desc(cfg, int(kk.max())),
        "cpu_baseline": {"value": round(v, 1), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args.record_traffic, args.config, args.plain_line, args.traffic_command)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
