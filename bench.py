"""Benchmark of the QSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
  prefill workloads: compressed-key pooling + indexer (query rotation, block
    scores, per-row top-k) + sparse attention over the selected K/V;
  decode workloads: ring pooling + decode indexer (scan + select) + split-KV
    sparse attention + combine.
The default run is the metric's own configurations: the line's workload is
the 128K-token prefill with heavy-tailed keys (B=1, T=131072, top-512, 16 q /
2 kv heads, bf16), and the same run measures the two decode workloads (8
sequences of 1M cached tokens, 64 sequences of 128K) and reports their
us/step under "decode".  --workload NAME measures one workload alone.  One
JSON line is printed by rank 0.  With N > 1 (torchrun) every rank runs its own replica of the
workload (QSA has no exchange step: replicas only), the timed region is
bracketed by barriers and the max over ranks is reported; value is the whole
job's throughput.

--impl reference times the CPU oracle (the only reference this method has) on
a bounded sample of the same workload on the host cores.
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

import torch  # noqa: E402

import workloads  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
# the metric's configurations: 128K-token prefill (the line), and the 1M and 128K decode steps
DEFAULT_WORKLOAD = "prefill_t128k_heavytail"
DEFAULT_DECODE = ("decode_b8_l1m_scale4", "decode_b64_l128k")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "block_sparse_attention_11_b200", "csrc")
# ncu summary holding the DRAM traffic of each roofline kernel, and the sources it was built from
_DECODE_SRC = ["k_decode_index.cu", "select.cuh", "common.cuh", "internal.h"]
TRAFFIC_PROFILE = {
    "prefill": [("attn_split_prefill_t128k.md", ["k_attn_tc.cu", "k_attn.cu", "common.cuh", "internal.h"])],
    "decode": [("decode_indexer_b64_l128k.md", _DECODE_SRC), ("decode_indexer_b64_l128k_fp8keys.md", _DECODE_SRC)],
}


def graph_stage_ms(fns, steps, dev):
    """Device time per call of each stage: the stage alone, `steps` calls back to
    back in its own CUDA graph (one untimed replay first), events around one
    replay.  The calls read the step's inputs and rewrite the same outputs, so
    repeating one stage is what the timed step graph does too."""
    out = []
    for fn in fns:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) / steps)
        del g
    return out


def source_digest(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kind, workload):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    summary is missing, covers another workload, or the kernel sources changed
    since it was captured."""
    for name, files in TRAFFIC_PROFILE[kind]:
        try:
            with open(os.path.join(PROFILES, name)) as f:
                txt = f.read()
        except OSError:
            continue
        fields = {}
        for line in txt.splitlines():
            if line.startswith("- ") and ": " in line:
                k, v = line[2:].split(": ", 1)
                fields[k.strip().strip("`")] = v.strip().strip("`")
        if fields.get("workload") != workload:
            continue
        try:
            if fields.get("source_sha256") != source_digest(files):
                return None
            return float(fields["traffic_bytes_per_launch"])
        except (KeyError, ValueError, OSError):
            return None
    return None


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- workload plumbing

class PrefillRunner:
    """Device buffers and one step of the prefill hot path."""

    def __init__(self, w, dev):
        import block_sparse_attention_11_b200 as qsa
        self.qsa = qsa
        self.w = w
        self.dev = dev
        self.x = workloads.make_prefill(w, device=dev)
        B, T = w.B, w.T
        dt = workloads.torch_dtype(w)
        # FP8 E4M3 K/V caches with per-tensor scales ("kv": "fp8"): the attention reads them
        self.kv8 = w.extra.get("kv") == "fp8"
        if self.kv8:
            self.x["k"], self.k_scale = workloads.to_e4m3(self.x["k"])
            self.x["v"], self.v_scale = workloads.to_e4m3(self.x["v"])
        self.rope = qsa.Rope(base=w.rope_base, pos_scale=w.pos_scale, rotary_dim=128)
        self.k_pool = torch.zeros(B, max(T // 4, 1), 128, dtype=dt, device=dev)
        # chunked prefill ("chunk" in extra): each chunk pools its keys into the growing
        # compressed cache, then selects and attends for its rows at offset q0 = c0
        self.chunks = chunk_bounds(T, w.extra.get("chunk"))
        if len(self.chunks) > 1:
            assert B == 1, "chunked prefill slices [1][T] inputs in place"
        rows = max(c1 - c0 for c0, c1 in self.chunks)
        self.sel = torch.empty(B, rows, w.top_k, dtype=torch.int32, device=dev)
        self.nsel = torch.empty(B, rows, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.x["q"])
        self.dt_code = 0 if w.dtype == "bf16" else 1
        ws = max(qsa.qsa_index_topk_prefill_workspace(B, c1 - c0, c0, w.top_k, 0, self.dt_code)
                 for c0, c1 in self.chunks)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        # the attention's workspace (the split's lists), allocated once
        wa = 0 if self.kv8 else max(qsa.qsa_sparse_attn_prefill_workspace(B, c1 - c0, w.top_k, w.Hq, w.Hkv, w.d,
                                                                          self.dt_code, q0=c0)
                                    for c0, c1 in self.chunks)
        self.ws_a = torch.empty(max(wa, 1), dtype=torch.uint8, device=dev)
        # the step's inputs (~200 MB at T=32K) do not all stay in L2, but the
        # flush keeps every timed step cold
        self.flush_between_steps = True
        self.use_graph = False        # three launches of milliseconds each: nothing to gain
        self.long_step = T > 262144   # steps of a second or more: shorter end-to-end runs

    def step(self, x=None, events=None):
        if len(self.chunks) > 1:
            return self.step_chunked(x, events)
        qsa, w = self.qsa, self.w
        x = x or self.x
        if events is not None:
            events[0].record()
        qsa.qsa_pool_keys_prefill(x["k_idx"], self.k_pool, rope=self.rope)
        if events is not None:
            events[1].record()
        qsa.qsa_index_topk_prefill(x["q_idx"], self.k_pool, self.sel, self.nsel, top_k=w.top_k, rope=self.rope,
                                   workspace=self.ws)
        if events is not None:
            events[2].record()
        if self.kv8:
            qsa.qsa_sparse_attn_prefill_kv8(x["q"], x["k"], x["v"], self.k_scale, self.v_scale, self.sel, self.nsel,
                                            self.out)
        else:
            qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], self.sel, self.nsel, self.out, workspace=self.ws_a)
        if events is not None:
            events[3].record()
        return self.out

    def step_chunked(self, x=None, events=None):
        """One chunked prefill of the whole prompt; per-chunk stage events are
        appended to `events` (after its first 4) for stage_times."""
        qsa, w = self.qsa, self.w
        x = x or self.x
        if events is not None:
            del events[4:]
            events[0].record()
        for c0, c1 in self.chunks:
            n = c1 - c0
            sel, nsel = self.sel[:, :n], self.nsel[:, :n]
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if events is not None else None
            if ev:
                ev[0].record()
            qsa.qsa_pool_keys_prefill(x["k_idx"][:, c0:c1], self.k_pool, pos0=c0, rope=self.rope)
            if ev:
                ev[1].record()
            qsa.qsa_index_topk_prefill(x["q_idx"][:, c0:c1], self.k_pool, sel, nsel, q0=c0, top_k=w.top_k,
                                       rope=self.rope, workspace=self.ws)
            if ev:
                ev[2].record()
            qsa.qsa_sparse_attn_prefill(x["q"][:, c0:c1], x["k"], x["v"], sel, nsel, self.out[:, c0:c1], q0=c0,
                                        workspace=self.ws_a)
            if ev:
                ev[3].record()
                events.extend(ev)
        if events is not None:
            events[1].record()
            events[2].record()
            events[3].record()
        return self.out

    def stage_times(self, events):
        """Stage milliseconds of one step: summed over chunks when chunked."""
        if len(events) <= 4:
            return [events[s].elapsed_time(events[s + 1]) for s in range(3)]
        t = [0.0, 0.0, 0.0]
        for j in range(4, len(events), 4):
            for s in range(3):
                t[s] += events[j + s].elapsed_time(events[j + s + 1])
        return t

    def launches_per_step(self):
        # per chunk: pooling, the indexer's kernels (query rotation, then scores + row select per row
        # chunk), the attention's kernels (lists + gather kernel + tiles per sequence and chunk of rows, or one)
        qsa, w = self.qsa, self.w
        n = 0
        for c0, c1 in self.chunks:
            n += 1 + qsa.qsa_index_topk_prefill_kernels(w.B, c1 - c0, c0, 0, self.dt_code)
            n += 1 if self.kv8 else qsa.qsa_sparse_attn_prefill_kernels(w.B, c1 - c0, w.top_k, w.Hq, w.Hkv, w.d,
                                                                        self.dt_code, q0=c0)
        return n

    def units(self):
        return self.w.B * self.w.T   # tokens

    def stage_names(self):
        return ["pool", "index_topk", "sparse_attn"]

    # algorithmic work (see the design notes): per-query gathered K/V bytes and flops
    def algorithmic(self):
        w = self.w
        T, K = w.T, w.top_k
        t = torch.arange(T, dtype=torch.float64)
        nb = torch.floor((t + 1) / 4)
        npos = torch.minimum(nb, torch.tensor(float(K))) * 4 + (t + 1 - 4 * nb)
        el = 1 if w.extra.get("kv") == "fp8" else 2                    # bytes per K/V element
        gather = float(npos.sum()) * w.Hkv * w.d * el * 2 * w.B       # K and V bytes gathered
        qo = 2.0 * T * w.Hq * w.d * 2 * w.B                            # q read + out write
        attn_flops = float(npos.sum()) * 4 * w.d * w.Hq * w.B
        pairs = float(nb.sum()) * w.B
        idx_flops = pairs * 2 * 128                                    # head-sum form of the linear score
        return dict(attn_bytes=gather + qo, attn_flops=attn_flops, idx_flops=idx_flops, pairs=pairs)

    def host_inputs(self):
        return {k: v.cpu().pin_memory() for k, v in self.x.items() if isinstance(v, torch.Tensor)}


def chunk_bounds(T, chunk):
    """[(c0, c1)] row ranges of a prefill done in chunks of `chunk` tokens (one range if None)."""
    chunk = int(chunk or T)
    return [(c0, min(c0 + chunk, T)) for c0 in range(0, T, chunk)]


class DecodeRunner:
    def __init__(self, w, dev):
        import block_sparse_attention_11_b200 as qsa
        self.qsa = qsa
        self.w = w
        self.dev = dev
        x = workloads.make_decode(w, device=dev)
        self.x = x
        dt = workloads.torch_dtype(w)
        B, L = w.B, w.T
        self.rope = qsa.Rope(base=w.rope_base, pos_scale=w.pos_scale, rotary_dim=128)
        self.cap = L // 4 + 1
        # compressed keys in the computation type, or FP8 E4M3 ("keys": "fp8")
        self.fp8 = w.extra.get("keys") == "fp8"
        self.kflags = qsa.QSA_KEYS_FP8 if self.fp8 else 0
        kdt = torch.float8_e4m3fn if self.fp8 else dt
        # FP8 E4M3 K/V caches with per-tensor scales ("kv": "fp8")
        self.kv8 = w.extra.get("kv") == "fp8"
        if self.kv8:
            x["k"], self.k_scale = workloads.to_e4m3(x["k"])
            x["v"], self.v_scale = workloads.to_e4m3(x["v"])
            torch.cuda.empty_cache()
        # paged caches ("page_tokens"): every sequence's pages scattered over a
        # shuffled pool, one page-table row per sequence
        self.pt = int(w.extra.get("page_tokens", 0))
        if self.pt:
            per_seq = (L + self.pt) // self.pt                 # positions 0 .. L
            num_pages = B * per_seq
            perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(w.seed))
            self.table = perm.view(B, per_seq).to(torch.int32).to(dev)
            pos = torch.arange(L + 1, device=dev)
            slots = (self.table[:, pos // self.pt].long() * self.pt + pos % self.pt)   # [B][L + 1]
            for name in ("k", "v"):
                pg = torch.empty(num_pages * self.pt, w.Hkv, w.d, dtype=dt, device=dev)
                pg[slots.reshape(-1)] = x[name][:, :L + 1].reshape(-1, w.Hkv, w.d)
                x[name] = pg
            torch.cuda.empty_cache()
            self.k_pool = torch.zeros(num_pages * self.pt // 4, 128, dtype=kdt, device=dev)
            qsa.qsa_pool_keys_prefill_paged(x["k_idx"], self.k_pool, self.table, self.pt, rope=self.rope,
                                            flags=self.kflags)
        else:
            self.k_pool = torch.zeros(B, self.cap, 128, dtype=kdt, device=dev)
            qsa.qsa_pool_keys_prefill(x["k_idx"], self.k_pool, rope=self.rope,      # the cache's compressed keys
                                      flags=self.kflags)
        self.ring = torch.zeros(B, 4, 128, dtype=dt, device=dev)
        del x["k_idx"]
        torch.cuda.empty_cache()
        self.sel = torch.empty(B, w.top_k, dtype=torch.int32, device=dev)
        self.nsel = torch.empty(B, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(x["q"])
        self.max_blocks = (L + 1) // 4
        self.ws_i = torch.zeros(qsa.qsa_index_topk_decode_workspace(B, self.max_blocks, w.top_k, self.kflags),
                                dtype=torch.uint8, device=dev)
        self.ws_a = torch.empty(qsa.qsa_sparse_attn_decode_workspace(B, w.Hq, w.d, w.top_k), dtype=torch.uint8,
                                device=dev)
        # a decode step streams the whole compressed-key cache and gathers from
        # K/V caches of several GB: inputs far larger than L2, no flush needed
        self.flush_between_steps = False
        # six launches of tens of microseconds: the step is replayed as a CUDA graph
        self.use_graph = True

    def step(self, x=None, events=None):
        x = x or self.x
        if events is not None:
            events[0].record()
        self.pool_ring(x)
        if events is not None:
            events[1].record()
        self.index(x)
        if events is not None:
            events[2].record()
        self.attend(x)
        if events is not None:
            events[3].record()
        return self.out

    def stage_fns(self):
        """The step's stages as separate calls (each repeatable on its own)."""
        return [self.pool_ring, self.index, self.attend]

    def pool_ring(self, x=None):
        """The step's new key into the ring; a completed block into the compressed cache."""
        qsa = self.qsa
        x = x or self.x
        if self.pt:
            qsa.qsa_pool_keys_decode_paged(x["k_idx_new"], self.ring, self.k_pool, self.table, self.pt,
                                           x["seq_len"], rope=self.rope, flags=self.kflags)
        else:
            qsa.qsa_pool_keys_decode(x["k_idx_new"], self.ring, self.k_pool, x["seq_len"], rope=self.rope,
                                     flags=self.kflags)

    def index(self, x=None):
        """The step's indexer call: scores and top-k into self.sel / self.nsel."""
        qsa, w = self.qsa, self.w
        x = x or self.x
        if self.pt:
            qsa.qsa_index_topk_decode_paged(x["q_idx"], self.k_pool, self.table, self.pt, x["seq_len"], self.sel,
                                            self.nsel, max_blocks=self.max_blocks, top_k=w.top_k, rope=self.rope,
                                            flags=self.kflags, workspace=self.ws_i)
        else:
            qsa.qsa_index_topk_decode(x["q_idx"], self.k_pool, x["seq_len"], self.sel, self.nsel,
                                      max_blocks=self.max_blocks, top_k=w.top_k, rope=self.rope, flags=self.kflags,
                                      workspace=self.ws_i)

    def attend(self, x=None):
        """The step's attention call alone, on the current self.sel / self.nsel."""
        qsa = self.qsa
        x = x or self.x
        if self.pt:
            qsa.qsa_sparse_attn_decode_paged(x["q"], x["k"], x["v"], self.table, self.pt, x["seq_len"], self.sel,
                                             self.nsel, self.out, workspace=self.ws_a)
        elif self.kv8:
            qsa.qsa_sparse_attn_decode_kv8(x["q"], x["k"], x["v"], self.k_scale, self.v_scale, x["seq_len"], self.sel,
                                           self.nsel, self.out, workspace=self.ws_a)
        else:
            qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], self.sel, self.nsel, self.out,
                                       workspace=self.ws_a)
        return self.out

    def launches_per_step(self):
        # ring pool, the indexer (one fused kernel, or scorer + select), attention, combine
        return 3 + self.qsa.qsa_index_topk_decode_kernels(self.w.B, self.max_blocks, self.kflags)

    def units(self):
        return self.w.B

    def stage_names(self):
        return ["pool_ring", "index_topk", "sparse_attn"]

    def algorithmic(self):
        w = self.w
        nb = (w.T + 1) // 4
        tail = (w.T + 1) - 4 * nb
        npos = min(nb, w.top_k) * 4 + tail
        kbytes = 1 if w.extra.get("keys") == "fp8" else 2
        el = 1 if w.extra.get("kv") == "fp8" else 2                    # bytes per K/V element
        idx_bytes = nb * 128 * kbytes + 4 * 128 * 2                   # compressed keys + indexer query
        kv_bytes = npos * w.Hkv * w.d * el * 2 + 2 * w.Hq * w.d * 2    # gathered K/V + q + out
        return dict(idx_bytes=idx_bytes * w.B, attn_bytes=kv_bytes * w.B, step_bytes=(idx_bytes + kv_bytes) * w.B)

    def host_inputs(self):
        keys = ["q_idx", "k_idx_new", "q", "seq_len"]
        return {k: self.x[k].cpu().pin_memory() for k in keys}


class DraftRunner:
    """IndexShare draft step: the selection of the capture row (the cache's
    new token) is made once, untimed; each timed step is the draft token's
    attention over that frozen selection plus the positions drafted since."""

    def __init__(self, w, dev):
        import block_sparse_attention_11_b200 as qsa
        self.qsa = qsa
        self.w = w
        self.dev = dev
        x = workloads.make_decode(w, device=dev)
        self.x = x
        dt = workloads.torch_dtype(w)
        B, L = w.B, w.T
        self.drafted = int(w.extra["drafted"])
        self.max_draft = int(w.extra["max_draft"])
        rope = qsa.Rope(base=w.rope_base, pos_scale=w.pos_scale, rotary_dim=128)
        cap = L // 4 + 1
        k_pool = torch.zeros(B, cap, 128, dtype=dt, device=dev)
        qsa.qsa_pool_keys_prefill(x["k_idx"], k_pool, rope=rope)
        ring = torch.zeros(B, 4, 128, dtype=dt, device=dev)
        qsa.qsa_pool_keys_decode(x["k_idx_new"], ring, k_pool, x["seq_len"], rope=rope)
        self.sel = torch.empty(B, w.top_k, dtype=torch.int32, device=dev)
        self.nsel = torch.empty(B, dtype=torch.int32, device=dev)
        qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], self.sel, self.nsel, max_blocks=(L + 1) // 4,
                                  top_k=w.top_k, rope=rope)      # the capture row's selection (setup)
        torch.cuda.synchronize()
        del x["k_idx"], k_pool
        torch.cuda.empty_cache()
        x["cap_len"] = x["seq_len"].clone()
        x["seq_len"] = x["seq_len"] + self.drafted
        self.out = torch.empty_like(x["q"])
        self.ws_a = torch.empty(qsa.qsa_sparse_attn_decode_shared_workspace(B, w.Hq, w.d, w.top_k, self.max_draft),
                                dtype=torch.uint8, device=dev)
        self.flush_between_steps = False      # K/V caches of several GB
        self.use_graph = True

    def step(self, x=None, events=None):
        qsa, w = self.qsa, self.w
        x = x or self.x
        if events is not None:
            events[0].record()
            events[1].record()
            events[2].record()
        qsa.qsa_sparse_attn_decode_shared(x["q"], x["k"], x["v"], x["seq_len"], x["cap_len"], self.sel, self.nsel,
                                          self.out, self.max_draft, workspace=self.ws_a)
        if events is not None:
            events[3].record()
        return self.out

    def launches_per_step(self):
        return 2   # attention, combine

    def units(self):
        return self.w.B

    def stage_names(self):
        return ["pool_ring_skipped", "index_skipped_frozen_selection", "sparse_attn"]

    def algorithmic(self):
        w = self.w
        t_c = w.T                                   # capture row (the cache's new token)
        nb = (t_c + 1) // 4
        npos = min(nb, w.top_k) * 4 + (t_c + self.drafted + 1 - 4 * nb)
        kv_bytes = npos * w.Hkv * w.d * 2 * 2 + 2 * w.Hq * w.d * 2
        return dict(attn_bytes=kv_bytes * w.B, step_bytes=kv_bytes * w.B, positions=npos)

    def host_inputs(self):
        keys = ["q", "seq_len", "cap_len"]
        return {k: self.x[k].cpu().pin_memory() for k in keys}


class DenseRunner:
    """Full causal decode attention over every cached position (the baseline
    QSA replaces), on the same caches as the QSA decode workloads."""

    def __init__(self, w, dev):
        import block_sparse_attention_11_b200 as qsa
        self.qsa = qsa
        self.w = w
        self.dev = dev
        x = workloads.make_decode(w, device=dev)
        del x["k_idx"]
        torch.cuda.empty_cache()
        self.x = x
        self.out = torch.empty_like(x["q"])
        self.ws = torch.empty(qsa.qsa_dense_attn_decode_workspace(w.B, w.Hq, w.d, x["k"].shape[1]),
                              dtype=torch.uint8, device=dev)
        self.flush_between_steps = False      # K/V caches of several GB
        self.use_graph = True

    def step(self, x=None, events=None):
        x = x or self.x
        if events is not None:
            events[0].record()
            events[1].record()
            events[2].record()
        self.qsa.qsa_dense_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], self.out, workspace=self.ws)
        if events is not None:
            events[3].record()
        return self.out

    def launches_per_step(self):
        return 2   # attention, combine

    def units(self):
        return self.w.B

    def stage_names(self):
        return ["no_pool", "no_index", "dense_attn"]

    def algorithmic(self):
        w = self.w
        npos = w.T + 1
        kv_bytes = npos * w.Hkv * w.d * 2 * 2 + 2 * w.Hq * w.d * 2
        return dict(attn_bytes=kv_bytes * w.B, step_bytes=kv_bytes * w.B, positions=npos)

    def host_inputs(self):
        return {k: self.x[k].cpu().pin_memory() for k in ["q", "seq_len"]}


class DensePrefillRunner:
    """Full causal prefill attention over every earlier position (the dense
    baseline the pages compare QSA's prefill with), on the QSA prefill
    workloads' q/k/v."""

    def __init__(self, w, dev):
        import block_sparse_attention_11_b200 as qsa
        self.qsa = qsa
        self.w = w
        self.dev = dev
        x = workloads.make_prefill(w, device=dev)
        self.x = {n: x[n] for n in ("q", "k", "v")}
        del x
        torch.cuda.empty_cache()
        self.out = torch.empty_like(self.x["q"])
        self.chunks = chunk_bounds(w.T, w.extra.get("chunk"))
        if len(self.chunks) > 1:
            assert w.B == 1, "chunked prefill slices [1][T] inputs in place"
        self.flush_between_steps = True
        self.use_graph = False
        self.long_step = w.T > 65536

    def step(self, x=None, events=None):
        x = x or self.x
        if events is not None:
            events[0].record()
            events[1].record()
            events[2].record()
        for c0, c1 in self.chunks:   # query rows c0 .. c1 - 1 over the cache up to each row
            self.qsa.qsa_dense_attn_prefill(x["q"][:, c0:c1], x["k"], x["v"], self.out[:, c0:c1], q0=c0)
        if events is not None:
            events[3].record()
        return self.out

    def launches_per_step(self):
        return len(self.chunks)

    def units(self):
        return self.w.B * self.w.T   # tokens

    def stage_names(self):
        return ["no_pool", "no_index", "dense_attn"]

    def algorithmic(self):
        w = self.w
        pairs = w.T * (w.T + 1) / 2 * w.B                              # (query, key) pairs, causal
        return dict(attn_flops=pairs * 4 * w.d * w.Hq)

    def host_inputs(self):
        return {k: v.cpu().pin_memory() for k, v in self.x.items()}


# ----------------------------------------------------------------------------- measurement

def flush_l2(buf):
    buf.add_(1.0)


def max_over_ranks(value, world, device):
    """The largest value over all ranks (the slowest rank's time); plain value at N=1."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms_per_step):
    """Whole-job units per second: every rank processes its own replica of the workload."""
    return units_per_rank * world / (ms_per_step / 1e3)


def run_ours(args, rank, world):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workloads.WORKLOADS[args.workload]
    runner = {"prefill": PrefillRunner, "decode": DecodeRunner, "draft": DraftRunner,
              "dense": DenseRunner, "dense_prefill": DensePrefillRunner}[w.kind](w, dev)
    flush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    qsa = runner.qsa
    for _ in range(args.warmup):
        runner.step()
    torch.cuda.synchronize()
    qsa.qsa_check_status()

    nst = 3
    graph = None
    if runner.use_graph:
        # The K timed steps (all library calls, preallocated workspaces) are
        # captured back to back in one CUDA graph, as a model's decode graph
        # holds its attention layers, so one graph launch is shared by K
        # complete steps; one untimed replay warms it up.
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            runner.step()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(args.steps):
                runner.step()
        graph.replay()
        torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    if graph is not None:
        events[0][0].record()
        graph.replay()                  # the K steps
        events[0][nst].record()
    else:
        for i in range(args.steps):
            if runner.flush_between_steps:
                flush_l2(flush)         # untimed: inputs start cold in L2
            runner.step(events=events[i])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    qsa.qsa_check_status()
    if graph is not None:
        step_ms = [events[0][0].elapsed_time(events[0][nst]) / args.steps] * args.steps
    else:
        step_ms = [events[i][0].elapsed_time(events[i][nst]) for i in range(args.steps)]
    stage_timing = "events between the stages of the timed steps"
    if graph is not None:
        # eager steps (per-stage events cannot sit inside the graph): their span is
        # reported as eager_step, and their stage split is the fallback below
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(args.steps)]
        for i in range(args.steps):
            runner.step(events=ev[i])
        torch.cuda.synchronize()
        eager_ms = sum(ev[i][0].elapsed_time(ev[i][nst]) for i in range(args.steps)) / args.steps
        stage_ms = [[ev[i][s].elapsed_time(ev[i][s + 1]) for i in range(args.steps)] for s in range(nst)]
        stage_timing = "events between the stages of eager steps (includes host launch gaps)"
        fns = getattr(runner, "stage_fns", None)
        if fns is not None:
            try:
                per = graph_stage_ms(fns(), args.steps, dev)
                stage_ms = [[t] * args.steps for t in per]
                stage_timing = "each stage alone, K calls back to back in one CUDA graph replay"
            except Exception as exc:   # keep the eager split
                print(f"bench: per-stage graph timing failed ({exc}); eager stage split", file=sys.stderr)
    else:
        eager_ms = None
        split = getattr(runner, "stage_times", None) or (lambda ev: [ev[s].elapsed_time(ev[s + 1])
                                                                      for s in range(nst)])
        per_step = [split(events[i]) for i in range(args.steps)]
        stage_ms = [[per_step[i][s] for i in range(args.steps)] for s in range(nst)]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps

    # end to end through the public API: pinned host inputs -> device -> QSA -> host result
    host = runner.host_inputs()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    out_host = torch.empty(runner.out.shape, dtype=runner.out.dtype, pin_memory=True)
    d2h = out_host.numel() * out_host.element_size()
    long_step = getattr(runner, "long_step", False)
    # steps of a second or more: one warm-up and one timed end-to-end step, serial only
    e2e_steps = 1 if long_step else max(3, min(args.steps, 10))
    e2e_warm = 1 if long_step else 2
    dev_x = dict(runner.x)

    def e2e_step():
        for k, v in host.items():
            dev_x[k] = v.to(dev, non_blocking=True)
        out = runner.step(x=dev_x)
        out_host.copy_(out, non_blocking=True)

    def timed(fn):
        for it in range(e2e_steps + e2e_warm):
            if it == e2e_warm:
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / e2e_steps

    e2e_serial_ms = timed(e2e_step)

    def e2e_pipelined(n):
        """n steps through the public API with the host copies of one step
        overlapping the compute of another: step i's inputs go host -> device on
        a copy stream into buffer set i % 2 while step i - 1 computes, and its
        output comes back on a third stream while step i + 1 computes.  Every
        step still copies all its inputs in and its result out."""
        bufs = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
        outs = [torch.empty_like(runner.out) for _ in range(2)]
        outs_h = [torch.empty(runner.out.shape, dtype=runner.out.dtype, pin_memory=True) for _ in range(2)]
        s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        comp = torch.cuda.current_stream(dev)
        ev = {n_: [torch.cuda.Event() for _ in range(2)] for n_ in ("h2d", "comp", "d2h")}
        keep_out = runner.out
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        s_h2d.wait_stream(comp)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(ev["comp"][b])        # step i - 2 has finished reading buffer set b
                for k, v in host.items():
                    bufs[b][k].copy_(v, non_blocking=True)
                ev["h2d"][b].record(s_h2d)
            comp.wait_event(ev["h2d"][b])
            if i >= 2:
                comp.wait_event(ev["d2h"][b])              # step i - 2's output has been read back
            xs = dict(runner.x)
            xs.update(bufs[b])
            runner.out = outs[b]
            runner.step(x=xs)
            ev["comp"][b].record(comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev["comp"][b])
                outs_h[b].copy_(outs[b], non_blocking=True)
                ev["d2h"][b].record(s_d2h)
        comp.wait_stream(s_d2h)
        e1.record(comp)
        torch.cuda.synchronize()
        runner.out = keep_out
        return e0.elapsed_time(e1) / n

    if long_step:
        e2e_pipe_ms = float("inf")
    else:
        e2e_pipelined(2)                # untimed: allocations and first launches
        e2e_pipe_ms = e2e_pipelined(e2e_steps)
    e2e_ms = min(e2e_serial_ms, e2e_pipe_ms)
    e2e_mode = "pipelined" if e2e_pipe_ms <= e2e_serial_ms else "serial"
    e2e_eager_ms = e2e_serial_ms
    if graph is not None:
        # the same public calls and copies (pinned host buffers), captured once and replayed
        for k, v in host.items():
            dev_x[k] = torch.empty_like(v, device=dev)
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            for k, v in host.items():
                dev_x[k].copy_(v, non_blocking=True)
            out = runner.step(x=dev_x)
            out_host.copy_(out, non_blocking=True)
        e2e_graph_ms = timed(g2.replay)
        del g2
        if e2e_graph_ms < e2e_ms:
            e2e_ms, e2e_mode = e2e_graph_ms, "graph"
    used_graph = graph is not None
    del graph

    pk, pk_kind = peaks()
    alg = runner.algorithmic()
    res = dict(n_gpus=world, steps=args.steps, warmup=args.warmup, ms_per_step=ms_per_step, dtype=w.dtype,
               data="synthetic", scaling="weak", vs_baseline=None, clocks=clocks,
               gpu_launches=runner.launches_per_step() * args.steps)
    stage_avg = {n: sum(v) / len(v) for n, v in zip(runner.stage_names(), stage_ms)}
    res["stage_ms"] = {k: round(v, 4) for k, v in stage_avg.items()}
    if eager_ms is not None:
        res["stage_ms"]["eager_step"] = round(eager_ms, 4)
    res["stage_timing"] = stage_timing
    if w.kind == "prefill":
        res.update(metric="QSA prefill tokens/s", unit="tokens/s", higher_is_better=True,
                   value=job_throughput(runner.units(), world, ms_per_step))
        res["e2e"] = dict(value=job_throughput(runner.units(), world, e2e_ms), unit="tokens/s", h2d_bytes_per_step=h2d,
                          d2h_bytes_per_step=d2h, mode=e2e_mode,
                          serial_value=job_throughput(runner.units(), world, e2e_serial_ms))
        attn_ms = stage_avg["sparse_attn"]
        attn_tf = alg["attn_flops"] / (attn_ms / 1e3) / 1e12
        peak_tf = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        res["roofline"] = dict(kernel="sparse_attn_prefill", bound="tensor", achieved=attn_tf, peak=peak_tf,
                               unit="TFLOP/s", frac=attn_tf / peak_tf,
                               traffic=profiled_traffic("prefill", w.name), peak_kind=pk_kind + " (sustained bf16)",
                               note="algorithmic flops = 4*d*Hq per selected position (4*nsel + tail per query) "
                                    "over the attention stage's CUDA-event time (its three kernels: block lists, "
                                    "gather kernel, tensor-core tiles); the bf16 sustained peak (a step of tens "
                                    "of ms)")
        flops = alg["attn_flops"] + alg["idx_flops"]
        tf = flops / (ms_per_step / 1e3) / 1e12
        res["tensor_roofline"] = dict(achieved=tf, peak=pk["bf16_tflops"], unit="TFLOP/s",
                                      frac=tf / pk["bf16_tflops"], peak_kind=pk_kind,
                                      note="indexer (2*128 flop per visible (query, block) pair) + attention "
                                           "(4*d*Hq flop per selected position) over the whole step")
        # per stage, the slower of its flops at the bf16 peak and its algorithmic bytes at the HBM
        # peak, summed, over the measured step (the attention's gathers are served from L2 when the
        # unique K/V fits there, so this can exceed 1)
        hbm, tens = pk["hbm_gbs"] * 1e9, pk["bf16_tflops"] * 1e12
        el = 2 if w.dtype == "bf16" else 4
        pool_b = w.B * w.T * 128 * el * 1.25
        idx_b = w.B * w.T * (4 * 128 * el + w.top_k * 4 + 4) + w.B * (w.T // 4) * 128 * el
        # the attention must read each K/V row of the sequence once from HBM (repeat gathers of a
        # block by other queries can be served by L2 or shared within a tile), plus q, out and sel
        attn_unique_b = w.B * w.T * (w.Hkv * w.d * el * 2 + 2 * w.Hq * w.d * 2 + w.top_k * 4)
        t_bound = (pool_b / hbm + max(alg["idx_flops"] / tens, idx_b / hbm)
                   + max(alg["attn_flops"] / tens, attn_unique_b / hbm))
        res["bound_aware"] = dict(bound_ms=t_bound * 1e3, frac=t_bound * 1e3 / ms_per_step,
                                  note="sum over pool, indexer, attention of max(flops / bf16 peak, bytes that "
                                       "must cross HBM / HBM peak), over the measured step time; the attention's "
                                       "HBM bytes are its unique inputs and outputs (each K/V row once)")
        res["config"] = dict(workload=w.name, B=w.B, T=w.T, top_k=w.top_k, Hq=w.Hq, Hkv=w.Hkv, d=w.d,
                             needles=w.needles, chunk=w.extra.get("chunk"),
                             l2="flushed between timed steps (256 MB write)",
                             parallelism=f"replicas x{world}")
    elif w.kind == "dense_prefill":
        res.update(metric=metric_name(w), unit="tokens/s", higher_is_better=True,
                   value=job_throughput(runner.units(), world, ms_per_step))
        res["e2e"] = dict(value=job_throughput(runner.units(), world, e2e_ms), unit="tokens/s", h2d_bytes_per_step=h2d,
                          d2h_bytes_per_step=d2h, mode=e2e_mode,
                          serial_value=job_throughput(runner.units(), world, e2e_serial_ms))
        tf = alg["attn_flops"] / (ms_per_step / 1e3) / 1e12
        peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        res["roofline"] = dict(kernel="dense_prefill_kernel", bound="tensor", achieved=tf, peak=peak,
                               unit="TFLOP/s", frac=tf / peak, traffic=None, peak_kind=pk_kind,
                               note="4*d*Hq flop per causal (query, key) pair over the step time; sustained bf16 "
                                    "peak (a step of tens of ms)")
        res["config"] = dict(workload=w.name, B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, d=w.d,
                             chunk=w.extra.get("chunk"), l2="flushed between timed steps (256 MB write)",
                             parallelism=f"replicas x{world}")
        if not args.no_library_context:
            res["library_context"] = library_dense_context(runner, alg["attn_flops"])
    elif w.kind in ("draft", "dense"):
        res.update(metric=metric_name(w), unit="us/step", higher_is_better=False, value=ms_per_step * 1e3)
        res["e2e"] = dict(value=e2e_ms * 1e3, unit="us/step", h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                          mode=e2e_mode, serial_value=e2e_eager_ms * 1e3)
        achieved = alg["attn_bytes"] / (ms_per_step / 1e3) / 1e9
        res["roofline"] = dict(kernel="sparse_attn_decode (frozen selection)" if w.kind == "draft"
                               else "dense causal decode attention", bound="hbm", achieved=achieved,
                               peak=pk["hbm_gbs"], unit="GB/s", frac=achieved / pk["hbm_gbs"], traffic=None,
                               peak_kind=pk_kind,
                               note=f"algorithmic bytes = {alg['positions']} gathered positions per sequence x Hkv x "
                                    f"d x 2 B x 2 + q/out; time = the graph-replayed step (attention + combine)")
        res["config"] = dict(workload=w.name, B=w.B, L=w.T, top_k=w.top_k, Hq=w.Hq, Hkv=w.Hkv, d=w.d,
                             drafted=w.extra.get("drafted", 0),
                             l2="inputs larger than L2 (K/V caches)", parallelism=f"replicas x{world}",
                             cuda_graph="the K timed steps captured in one graph")
    else:
        res.update(metric="QSA decode us/step", unit="us/step", higher_is_better=False,
                   value=ms_per_step * 1e3)
        res["e2e"] = dict(value=e2e_ms * 1e3, unit="us/step", h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                          mode=e2e_mode, serial_value=e2e_eager_ms * 1e3)
        idx_ms = stage_avg["index_topk"]
        achieved = alg["idx_bytes"] / (idx_ms / 1e3) / 1e9
        res["roofline"] = dict(kernel="decode indexer (scorer + select)", bound="hbm", achieved=achieved,
                               peak=pk["hbm_gbs"], unit="GB/s", frac=achieved / pk["hbm_gbs"],
                               traffic=profiled_traffic("decode", w.name), peak_kind=pk_kind,
                               note="algorithmic bytes = every compressed key of every sequence (ceil(L/4) x 128 x "
                                    f"{1 if w.extra.get('keys') == 'fp8' else 2} B) + indexer query; time = the "
                                    "index stage (the fused scorer-select kernel, or scorer + select) as "
                                    "stage_timing states; traffic = the indexer kernels' DRAM bytes per call")
        step_ach = alg["step_bytes"] / (ms_per_step / 1e3) / 1e9
        res["step_roofline"] = dict(bound="hbm", achieved=step_ach, peak=pk["hbm_gbs"], unit="GB/s",
                                    frac=step_ach / pk["hbm_gbs"], peak_kind=pk_kind,
                                    note="whole decode step (graph replay): compressed keys + gathered K/V + q/o "
                                         "bytes over the step time")
        res["config"] = dict(workload=w.name, B=w.B, L=w.T, top_k=w.top_k, Hq=w.Hq, Hkv=w.Hkv, d=w.d,
                             pos_scale=w.pos_scale, l2="inputs larger than L2 (compressed-key cache and K/V caches)",
                             parallelism=f"replicas x{world}", cuda_graph="the K timed steps captured in one graph")
    return res


def library_dense_context(runner, flops, reps=2):
    """Context for the dense comparator, not a figure of this library: cuDNN's
    fused causal attention (torch SDPA, cuDNN backend) on the same q/k/v as one
    whole-sequence call per group of q heads (each call's q at most 2^28
    elements), timed with CUDA events after one untimed call."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    w = runner.w
    q, k, v = (runner.x[n] for n in ("q", "k", "v"))
    B, T, Hq, d = q.shape
    G = Hq // w.Hkv
    hq_call = max(1, min(Hq, (1 << 28) // (B * T * d)))
    while Hq % hq_call or (hq_call % G and G % hq_call):
        hq_call -= 1
    out = torch.empty_like(q)

    def run():
        for h0 in range(0, Hq, hq_call):
            kv0, kv1 = h0 // G, (h0 + hq_call - 1) // G + 1
            o = F.scaled_dot_product_attention(q[:, :, h0:h0 + hq_call].transpose(1, 2),
                                               k[:, :, kv0:kv1].transpose(1, 2), v[:, :, kv0:kv1].transpose(1, 2),
                                               is_causal=True, enable_gqa=True)
            out[:, :, h0:h0 + hq_call] = o.transpose(1, 2)

    try:
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            run()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                run()
            e1.record()
            torch.cuda.synchronize()
    except Exception as e:   # backend unavailable in this torch or on this device
        return dict(library="cuDNN fused attention via torch SDPA", unavailable=repr(e)[:160])
    ms = e0.elapsed_time(e1) / reps
    tail = slice(max(0, T - 2048), T)
    diff = (out[:, tail].float() - runner.out[:, tail].float()).abs().max().item()
    return dict(library="cuDNN fused attention via torch SDPA (context only; not this library)",
                ms_per_step=ms, tokens_per_s=B * T / (ms / 1e3), tflops=flops / (ms / 1e3) / 1e12,
                calls_per_step=Hq // hq_call, max_abs_diff_vs_ours_last_2048_rows=diff,
                note="whole-sequence causal calls (the same (query, key) pairs as the chunked steps)")


# ----------------------------------------------------------------------------- CPU oracle arm

ORACLE_EXTRA = {}   # figures beside the main oracle timing (the one-thread rate), per run


def run_oracle_sample(w, budget_s=15.0, seed=0):
    """Time the CPU oracle on a bounded sample of the workload; returns
    (value in the workload's unit, sample description, threads)."""
    import numpy as np

    import oracle
    nthreads = os.cpu_count() or 1
    if w.kind == "prefill":
        x = workloads.make_prefill(w, device="cpu")
        dequant_kv(w, x)
        q_idx = x["q_idx"][0].float().numpy()
        k_raw = x["k_idx"][0].float().numpy()
        q, k, v = (x[n][0].float().numpy() for n in ("q", "k", "v"))
        t0 = time.perf_counter()
        kp = oracle.pool_keys(k_raw, base=w.rope_base, pos_scale=w.pos_scale, store_bf16=w.dtype == "bf16")
        t_pool = time.perf_counter() - t0
        rng = np.random.default_rng(seed)
        done, elapsed, n = 0, 0.0, 64
        while elapsed < budget_s and done < w.T:
            rows = rng.integers(0, w.T, n)
            t0 = time.perf_counter()
            oracle.prefill_rows(rows, q_idx=q_idx, k_pool=kp, top_k=w.top_k, base=w.rope_base,
                                pos_scale=w.pos_scale, store_bf16=w.dtype == "bf16", q=q, k=k, v=v, Hq=w.Hq,
                                Hkv=w.Hkv, d=w.d, nthreads=nthreads)
            dt = time.perf_counter() - t0
            elapsed += dt
            done += n
            n = min(4096, n * 2)
        per_row = elapsed / done
        total = t_pool + per_row * w.T * w.B
        value = w.T * w.B / total
        # one thread on a short sample of the same rows' distribution
        rows1 = rng.integers(0, w.T, 32)
        t0 = time.perf_counter()
        oracle.prefill_rows(rows1, q_idx=q_idx, k_pool=kp, top_k=w.top_k, base=w.rope_base,
                            pos_scale=w.pos_scale, store_bf16=w.dtype == "bf16", q=q, k=k, v=v, Hq=w.Hq,
                            Hkv=w.Hkv, d=w.d, nthreads=1)
        per_row1 = (time.perf_counter() - t0) / len(rows1)
        ORACLE_EXTRA["value_1thread"] = w.T * w.B / (t_pool + per_row1 * w.T * w.B)
        ORACLE_EXTRA["sample_1thread"] = "32 uniformly drawn rows, one thread, extrapolated the same way"
        sample = (f"{done} uniformly drawn query rows of the {w.T}-token workload (full indexer scan, top-k, "
                  f"attention per row) + pooling of all keys; extrapolated per row to all rows")
        return value, sample, nthreads, "tokens/s"
    if w.kind == "dense_prefill":   # textbook causal attention of sampled rows, per row cost ~ its position
        x = workloads.make_prefill(w, device="cpu")
        q, k, v = (x[n][0].float().numpy() for n in ("q", "k", "v"))
        rng = np.random.default_rng(seed)
        done_pos, elapsed, n = 0.0, 0.0, 8
        while elapsed < budget_s:
            rows = rng.integers(0, w.T, n)
            t0 = time.perf_counter()
            oracle.dense_rows(rows, q=q, k=k, v=v, Hq=w.Hq, Hkv=w.Hkv, d=w.d, nthreads=nthreads)
            elapsed += time.perf_counter() - t0
            done_pos += float((rows + 1).sum())
            n = min(1024, n * 2)
        total = elapsed / done_pos * (w.T * (w.T + 1) / 2) * w.B       # extrapolated by causal positions
        return (w.T * w.B / total, "uniformly drawn query rows (textbook attention over their causal prefix); "
                "extrapolated by positions to all rows", nthreads, "tokens/s")
    if w.kind == "dense":   # textbook causal attention of one sequence's new token
        x = workloads.make_decode(w, device="cpu", B=1)
        q, k, v = x["q"].float().numpy(), x["k"][0].float().numpy(), x["v"][0].float().numpy()
        t = int(x["seq_len"][0]) - 1
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle.dense_rows([0], q=q, k=k, v=v, Hq=w.Hq, Hkv=w.Hkv, d=w.d, q0=t, nthreads=nthreads)
            reps += 1
            if time.perf_counter() - t0 > min(budget_s, 5.0):
                break
        value = (time.perf_counter() - t0) / reps * w.B * 1e6
        return value, f"{reps} steps of one {w.T}-token sequence, scaled to B={w.B}", nthreads, "us/step"
    # decode: a subset of sequences at full length
    x = workloads.make_decode(w, device="cpu", B=1)
    dequant_kv(w, x)
    kr = x["k_idx"][0].float().numpy()
    kp = oracle.pool_keys(kr, base=w.rope_base, pos_scale=w.pos_scale, store_bf16=True,
                          store_fp8=w.extra.get("keys") == "fp8")
    q, k, v = x["q"].float().numpy(), x["k"].float().numpy(), x["v"].float().numpy()
    seq_len = x["seq_len"].numpy()
    cap_len = None
    if w.kind == "draft":                # the drafted positions follow the capture row
        cap_len = seq_len.copy()
        seq_len = seq_len + int(w.extra["drafted"])
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.decode(x["q_idx"].float().numpy(), kp[None], seq_len, cap_len=cap_len, q=q, k=k, v=v,
                      top_k=w.top_k, base=w.rope_base, pos_scale=w.pos_scale, Hq=w.Hq, Hkv=w.Hkv, d=w.d,
                      nthreads=nthreads)
        reps += 1
        if time.perf_counter() - t0 > min(budget_s, 5.0):
            break
    per_seq = (time.perf_counter() - t0) / reps
    value = per_seq * w.B * 1e6          # a step of all B sequences, us
    sample = f"{reps} decode steps of one {w.T}-token sequence, scaled to B={w.B}"
    if w.kind == "draft":
        sample += " (the oracle selects for the capture row on every step: it takes no frozen selection)"
    return value, sample, nthreads, "us/step"


def dequant_kv(w, x):
    """FP8 K/V workloads: the oracle reads the dequantized caches."""
    if w.extra.get("kv") == "fp8":
        for n in ("k", "v"):
            c, sc = workloads.to_e4m3(x[n])
            x[n] = c.float() * sc


def metric_name(w):
    return {"prefill": "QSA prefill tokens/s", "decode": "QSA decode us/step",
            "draft": "QSA IndexShare draft step us/step", "dense": "full causal decode attention us/step",
            "dense_prefill": "full causal prefill attention tokens/s"}[w.kind]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=sorted(workloads.WORKLOADS),
                    help="one workload alone (default: the 128K prefill line with both decode workloads)")
    ap.add_argument("--no-decode", action="store_true", help="default run: skip the two decode workloads")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-library-context", action="store_true",
                    help="full-attention workloads: skip timing cuDNN's attention beside ours")
    ap.add_argument("--batch", type=int, default=None, help="override B (smaller profiling case)")
    ap.add_argument("--tokens", type=int, default=None, help="override T / cache length (smaller profiling case)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    with_decode = args.workload is None and not args.no_decode
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return                      # the CPU oracle arm runs on rank 0 only
    if world > 1 and args.impl != "reference":
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    w = workloads.WORKLOADS[args.workload]
    if args.batch or args.tokens:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch or w.B, T=args.tokens or w.T, name=w.name + "_profile_case")
        workloads.WORKLOADS[w.name] = w
        args.workload = w.name

    if args.impl == "reference":
        if rank == 0:
            value, sample, threads, unit = run_oracle_sample(w, budget_s=args.cpu_budget)
            line = dict(impl="reference", metric=metric_name(w), value=value, unit=unit,
                        higher_is_better=w.kind in ("prefill", "dense_prefill"),
                        n_gpus=args.gpus, steps=args.steps, warmup=args.warmup, dtype=w.dtype, data="synthetic",
                        config=dict(workload=w.name), vs_baseline=None,
                        cpu_baseline=dict(value=value, unit=unit, cores=threads, kind="oracle", sample=sample,
                                          **ORACLE_EXTRA),
                        e2e=dict(value=value, unit=unit, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
            print(json.dumps(line), flush=True)
        return

    res = run_ours(args, rank, world)
    if rank == 0 and not args.no_cpu_baseline:
        value, sample, threads, unit = run_oracle_sample(w, budget_s=args.cpu_budget)
        res["cpu_baseline"] = dict(value=value, unit=unit, cores=threads, kind="oracle", sample=sample,
                                   **ORACLE_EXTRA)
    if with_decode:
        # the metric's decode half, in the same run: each decode workload timed as its own step
        res["decode"] = {}
        for name in DEFAULT_DECODE:
            torch.cuda.empty_cache()
            sub_args = argparse.Namespace(**vars(args))
            sub_args.workload = name
            sub = run_ours(sub_args, rank, world)
            if rank == 0 and not args.no_cpu_baseline:
                ORACLE_EXTRA.clear()
                value, sample, threads, unit = run_oracle_sample(workloads.WORKLOADS[name],
                                                                 budget_s=min(args.cpu_budget, 6.0))
                sub["cpu_baseline"] = dict(value=value, unit=unit, cores=threads, kind="oracle", sample=sample)
            keep = ["metric", "value", "unit", "ms_per_step", "higher_is_better", "config", "roofline",
                    "step_roofline", "e2e", "cpu_baseline", "gpu_launches", "clocks", "stage_ms", "stage_timing"]
            res["decode"][name] = {k: sub[k] for k in keep if k in sub}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        order = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                 "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "l2_roofline", "tensor_roofline",
                 "bound_aware", "step_roofline",
                 "e2e",
                 "cpu_baseline", "gpu_launches", "clocks", "stage_ms", "stage_timing", "library_context", "decode"]
        line = {k: res[k] for k in order if k in res}
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
