#!/usr/bin/env python3
"""Benchmark of the HEAL hot path on B200 (one JSON line on stdout, rank 0).

One step = one pass of every hot-path kernel over one batch of seeded synthetic input:
  * compensated GEMM, prefill linear: X[4096x4096] (1% outlier columns x20) . W[4096x14336],
    both FP32, split to FP16 hi/lo inside the kernel                      (headline)
  * compensated GEMM, decode: X[M x 4096] . W[4096x4096] for M = 1, 8, 64
  * INT16 KV writer: Q [8,1,32,128], K and V [8,8192,8,128] bf16 -> INT16 caches
  * INT16 decode attention over the 8192-token caches, 32 query / 8 KV heads
Each part is captured once into a CUDA graph from the library calls and replayed every step;
CUDA events on the replay stream time every part; `value` is the prefill GEMM's effective
TFLOP/s (2MNK / time).  The e2e figure calls the library directly, with host buffers.  All inputs are larger than L2 or are separate
buffers with more than 1 GB of other traffic between their reuses, so each kernel reads
cold from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (torchrun): every rank runs the same step on its own seeded shard, no
collective on the data path ("weak" scaling); timings are the max over ranks.
"""
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

METRIC = "compensated-GEMM effective TFLOP/s (% of 16-bit TC peak); INT16-KV attn GB/s"
PREFILL = (4096, 4096, 14336)
DECODE_M = (1, 8, 64)
CHAIN = 8             # decode GEMMs issued back to back in the chain part
KV = dict(B=8, T=8192, Hkv=8, Hq=32, D=128)
L2_CLEAN_BYTES = 256 * 1024 * 1024
REF_COPY_BYTES = 4 * 4096 * 4096          # bytes a decode GEMM reads (FP32 4096 x 4096 weights)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the active clock-event (throttle) reasons every ~10 ms
    through NVML while the timed region runs (read-only queries)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        except Exception as exc:
            self.error = repr(exc)
            self.nv = None
        return self

    def _poll(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), int(get_reasons(self.h))))
            except Exception as exc:
                self.error = repr(exc)
                return
            time.sleep(0.01)

    def __exit__(self, *exc):
        self._stop.set()
        if self.nv is not None:
            self.t.join(timeout=2)

    def summary(self):
        loaded = [(mhz, bits) for mhz, bits in self.samples if not bits & 0x1]
        reasons = sorted({name for _, bits in loaded for b, name in self.REASONS.items() if bits & b})
        out = {"sm_mhz": statistics.median([m for m, _ in loaded]) if loaded else None,
               "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(loaded),
               "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


# --------------------------------------------------------------------------- workload
class Workload:
    """Device-resident inputs and outputs of one rank's step."""

    def __init__(self, torch, heal, synthetic, dev, seed_offset=0, only=None):
        """only: None for the whole step, or one part (a profiling case allocates only its buffers)."""
        self.torch, self.heal = torch, heal
        self.only = only
        M, K, N = PREFILL
        so = seed_offset
        # L2 cleaning before every part of a step (outside the part's events): a buffer
        # larger than L2 (126 MB) is written, then two others are read, so that each part
        # starts with none of its inputs in L2, without another part's dirty lines, whose
        # write-back it would otherwise pay for, and after the write-backs of the flush's
        # own lines (evicted by the first read) have drained during the second.
        self.l2_w = torch.zeros(L2_CLEAN_BYTES // 4, device=dev)
        self.l2_r = torch.zeros(L2_CLEAN_BYTES // 4, device=dev)
        self.l2_r2 = torch.zeros(L2_CLEAN_BYTES // 4, device=dev)
        self.l2_acc = torch.zeros(1, device=dev)
        need = lambda part: only is None or only == part or (part == "kv_writer" and only == "attention")
        if need("prefill"):
            X, W = synthetic.gemm_prefill(M=M, K=K, N=N, seed_x=0 + so, seed_w=1 + so)
            self.X, self.W = X.to(dev), W.to(dev)
            self.C = torch.empty(M, N, device=dev)
            # scratch for the optional split pass over B (timed apart from the step)
            self.wsp = torch.empty(heal.heal_gemm_workspace_bytes(M, N, K, b_split_pass=True), dtype=torch.uint8,
                                   device=dev)
            # the same weights split once (static weights held as hi / lo)
            self.Whi = torch.empty(self.W.shape, dtype=torch.int16, device=dev)
            self.Wlo = torch.empty(self.W.shape, dtype=torch.int16, device=dev)
            heal.heal_split(self.W, self.Whi, self.Wlo)
            # the same weights held as FP16 values (two products: only X is split)
            self.W16 = self.W.half()
        self.dec = []
        if need("decode"):
            # a plain device copy moving as many bytes as one decode GEMM reads (32 MB read,
            # 32 MB written): the single-launch streaming time at this size, timed like the
            # decode parts (torch's copy kernel, not this library's; context only)
            self.ref_src = torch.zeros(REF_COPY_BYTES // 8, device=dev)
            self.ref_dst = torch.zeros(REF_COPY_BYTES // 8, device=dev)
            # and a plain read of that many bytes (a one-dimensional sum)
            self.ref_read = torch.zeros(REF_COPY_BYTES // 4, device=dev)
            self.ref_acc = torch.zeros(1, device=dev)
            for i, m in enumerate(DECODE_M):
                Xd, Wd = synthetic.gemm_decode(m, seed_x=0 + so, seed_w=1 + so + 10 * (i + 1))
                ws = torch.empty(max(1, heal.heal_gemm_workspace_bytes(m, 4096, 4096, heal.TILE_SKINNY_SPLITK) // 4),
                                 device=dev)
                Wd = Wd.to(dev)
                # the same weights split once (as a deployment would at load time): hi / lo
                whi = torch.empty(Wd.shape, dtype=torch.int16, device=dev)
                wlo = torch.empty(Wd.shape, dtype=torch.int16, device=dev)
                heal.heal_split(Wd, whi, wlo)
                self.dec.append((m, Xd.to(dev), Wd, torch.empty(m, 4096, device=dev), ws, whi, wlo))
            # a chain of CHAIN decode GEMMs with distinct weights, each one's output the next
            # one's input, issued back to back as a decoder issues its projections
            self.chain = []
            for i in range(CHAIN):
                Wc = synthetic.normal((4096, 4096), seed=500 + so + i, std=0.02).to(dev)
                chi = torch.empty(Wc.shape, dtype=torch.int16, device=dev)
                clo = torch.empty(Wc.shape, dtype=torch.int16, device=dev)
                heal.heal_split(Wc, chi, clo)
                self.chain.append((Wc, chi, clo, torch.empty(1, 4096, device=dev)))
            # the same weights held as FP16 values (the two-product form: only activations split)
            self.dec16 = [(m, Xd, chi16, Cd, ws) for (m, Xd, Wd, Cd, ws, whi, wlo), chi16 in
                          zip(self.dec, [Wd.half() for (m, Xd, Wd, Cd, ws, whi, wlo) in self.dec])]
            self.chain16 = [Wc.half() for (Wc, chi, clo, Cc) in self.chain]
            self.chain_x = synthetic.normal((1, 4096), seed=600 + so).to(dev)
            self.chain_ws = torch.empty(heal.heal_gemm_workspace_bytes(1, 4096, 4096, heal.TILE_SKINNY_SPLITK) // 4,
                                        device=dev)
        if need("kv_writer"):
            B, T, Hkv, Hq, D = KV["B"], KV["T"], KV["Hkv"], KV["Hq"], KV["D"]
            Qb, Kb, Vb = synthetic.kv_decode(B=B, T=T, Hkv=Hkv, Hq=Hq, D=D, seeds=(2 + so, 3 + so, 4 + so))
            self.Qb, self.Kb, self.Vb = Qb.to(dev), Kb.to(dev), Vb.to(dev)
            i16, f32 = torch.int16, torch.float32
            self.qc = torch.empty(B, Hq, 1, D, dtype=i16, device=dev)
            self.qs = torch.empty(B, Hq, 1, dtype=f32, device=dev)
            self.kc = torch.empty(B, Hkv, T, D, dtype=i16, device=dev)
            self.ks = torch.empty(B, Hkv, T, dtype=f32, device=dev)
            self.vc = torch.empty(B, Hkv, T, D, dtype=i16, device=dev)
            self.vs = torch.empty(B, Hkv, T, dtype=f32, device=dev)
            self.kv_len = torch.full((B,), T, dtype=torch.int32, device=dev)
            self.out = torch.empty(B, Hq, 1, D, device=dev)
            self.aws = torch.empty(heal.heal_attention_workspace_bytes(B, Hq, 1, T) // 4, device=dev)

    # algorithmic bytes / flops per launch (what the method must touch, once)
    @staticmethod
    def units():
        M, K, N = PREFILL
        B, T, Hkv, Hq, D = KV["B"], KV["T"], KV["Hkv"], KV["Hq"], KV["D"]
        kv_elems = B * T * Hkv * D
        return {
            "prefill_flop_eff": 2.0 * M * N * K,
            "prefill_flop_mma": 3 * 2.0 * M * N * K,
            "decode_bytes": {m: 4.0 * (4096 * 4096 + m * 4096 + m * 4096) for m in DECODE_M},
            "chain_bytes": CHAIN * 4.0 * (4096 * 4096 + 2 * 4096),
            "decode16_bytes": {m: 2.0 * 4096 * 4096 + 4.0 * (m * 4096 + m * 4096) for m in DECODE_M},
            "chain16_bytes": CHAIN * (2.0 * 4096 * 4096 + 8.0 * 4096),
            "kv_writer_bytes": 2 * (2 * kv_elems + 2 * kv_elems + 4 * B * Hkv * T) + (2 + 2) * B * Hq * D + 4 * B * Hq,
            "attn_bytes": 2 * (2 * kv_elems + 4 * B * Hkv * T) + 2 * B * Hq * D + 4 * B * Hq + 4 * B * Hq * D,
        }

    def parts(self):
        """The parts of one step as (name, callable launching that part's library calls)."""
        h = self.heal
        out = []
        only = self.only
        # Independent parts, each timed after an L2 clean (run_graphs): the KV writer (which
        # fills the caches attention reads), the prefill product, attention, the decode GEMMs.
        if only in (None, "kv_writer", "attention"):
            out.append(("kv_writer", lambda: (h.heal_kv_quantize_int16(self.Qb, self.qc, self.qs),
                                              h.heal_kv_quantize_int16(self.Kb, self.kc, self.ks),
                                              h.heal_kv_quantize_int16(self.Vb, self.vc, self.vs))))
        if only in (None, "prefill"):
            out.append(("prefill", lambda: self.prefill()))
        if only in (None, "attention"):
            out.append(("attention", lambda: h.heal_attention_int16(
                self.qc, self.qs, self.kc, self.ks, self.vc, self.vs, self.kv_len, KV["D"] ** -0.5, self.out,
                self.aws)))
        if only in (None, "decode"):
            for (m, Xd, Wd, Cd, ws, whi, wlo) in self.dec:
                out.append((f"decode{m}", lambda Xd=Xd, Wd=Wd, Cd=Cd, ws=ws: h.heal_gemm_compensated(
                    Xd, Wd, Cd, workspace=ws)))
            for (m, Xd, Wd, Cd, ws, whi, wlo) in self.dec:
                out.append((f"decode{m}_presplit", lambda Xd=Xd, whi=whi, wlo=wlo, Cd=Cd, ws=ws:
                            h.heal_gemm_compensated(Xd, whi, Cd, b_lo=wlo, workspace=ws)))
            for (m, Xd, W16, Cd, ws) in self.dec16:
                out.append((f"decode{m}_w16", lambda Xd=Xd, W16=W16, Cd=Cd, ws=ws: h.heal_gemm_compensated(
                    Xd, W16, Cd, workspace=ws, b_16bit=True)))
            out.append(("decode1_chain", lambda: self.run_chain(False)))
            out.append(("decode1_chain_presplit", lambda: self.run_chain(True)))
            out.append(("decode1_chain_w16", lambda: self.run_chain16()))
            out.append(("ref_copy_67MB", lambda: self.ref_dst.copy_(self.ref_src)))
            out.append(("ref_read_67MB", lambda: self.torch.sum(self.ref_read, dim=0, out=self.ref_acc[0])))
        return out

    def prefill(self):
        # FP32 A and B, both split by the producer-side split warps inside the kernel
        self.heal.heal_gemm_compensated(self.X, self.W, self.C)

    def run_chain(self, presplit):
        a = self.chain_x
        for (Wc, chi, clo, Cc) in self.chain:
            if presplit:
                self.heal.heal_gemm_compensated(a, chi, Cc, b_lo=clo, workspace=self.chain_ws, b_static=True)
            else:
                self.heal.heal_gemm_compensated(a, Wc, Cc, workspace=self.chain_ws, b_static=True)
            a = Cc

    def run_chain16(self):
        a = self.chain_x
        for (Wc, chi, clo, Cc), W16 in zip(self.chain, self.chain16):
            self.heal.heal_gemm_compensated(a, W16, Cc, workspace=self.chain_ws, b_static=True, b_16bit=True)
            a = Cc

    def capture(self, stream):
        """One CUDA graph per part, captured from the library calls (replays launch the same
        kernels with the same arguments, without Python or driver overhead per call)."""
        torch = self.torch
        self.graphs = []
        for name, fn in self.parts():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            self.graphs.append((name, g))

    def l2_clean(self):
        self.l2_w.zero_()
        self.torch.sum(self.l2_r, dim=0, out=self.l2_acc[0])
        self.torch.sum(self.l2_r2, dim=0, out=self.l2_acc[0])

    def run_graphs(self, ev=None):
        for name, g in self.graphs:
            self.l2_clean()
            if ev is not None:
                ev[name][0].record()
            g.replay()
            if ev is not None:
                ev[name][1].record()

    def run(self, ev=None):
        """One step, eagerly (the warm-up before capture).  ev: dict name -> (start, end) CUDA
        events, recorded around each part."""
        for name, fn in self.parts():
            if ev is not None:
                ev[name][0].record()
            fn()
            if ev is not None:
                ev[name][1].record()

    LAUNCHES_PER_STEP = 1 + 3 * 2 * len(DECODE_M) + 3 * 2 * CHAIN + 3 + 2


def decoder_section(torch, heal, synthetic, dev, stream, prompt_len=512, steps=128):
    """2-layer random-init decoder (hidden 4096, 32q/8kv heads, FFN 14336, vocab 128256):
    time of the 512-token prefill and per greedy decode step, and a bitwise repeat check."""
    from error_compensated_gemm_b200.decoder import Decoder
    cfg = synthetic.DecoderConfig(max_pos=prompt_len + steps + 64)
    w = synthetic.decoder_weights(cfg)
    prompt = synthetic.prompt_ids(prompt_len, cfg.vocab).to(dev)
    dec = Decoder(cfg, w, dev, max_len=prompt_len + steps + 64)
    del w
    t_ref, _ = dec.generate(prompt, 8)                      # warm-up
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    tok = torch.empty(steps, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    dec.pos_len = 0
    ev[0].record(stream)
    logits = dec.forward(prompt)
    ev[1].record(stream)
    for s in range(steps):
        heal.heal_argmax(logits, tok[s:s + 1].view(1))
        if s + 1 < steps:
            logits = dec.forward(tok[s:s + 1])
    ev[2].record(stream)
    torch.cuda.synchronize()
    t_again, _ = dec.generate(prompt, steps)
    torch.cuda.synchronize()
    pre = ev[0].elapsed_time(ev[1])
    per = ev[1].elapsed_time(ev[2]) / steps
    # the same greedy steps captured once as a CUDA graph (the way a serving loop runs
    # decode): after an eager prefill, one replay runs all steps without host round trips
    cap = torch.cuda.Stream()
    tok_g = torch.empty(steps, dtype=torch.int32, device=dev)
    dec.pos_len = 0
    logits0 = dec.forward(prompt)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        lg = logits0
        for s in range(steps):
            heal.heal_argmax(lg, tok_g[s:s + 1].view(1))
            if s + 1 < steps:
                lg = dec.forward(tok_g[s:s + 1])
    dec.pos_len = 0
    dec.forward(prompt)                                         # caches back to the post-prefill state
    torch.cuda.synchronize()
    ev[1].record(stream)
    graph.replay()
    ev[2].record(stream)
    torch.cuda.synchronize()
    per_graph = ev[1].elapsed_time(ev[2]) / steps
    same = bool(torch.equal(tok, tok_g))
    del graph
    return {"prefill_ms": pre, "decode_ms_per_token": per, "decode_tokens_per_s": 1e3 / per,
            "decode_graph_ms_per_token": per_graph, "decode_graph_tokens_per_s": 1e3 / per_graph,
            "prompt": prompt_len, "steps": steps, "bitwise_repeat": bool(torch.equal(tok, t_again)),
            "graph_tokens_equal_eager": same,
            "note": "decode_ms_per_token: each step launched from Python; decode_graph_ms_per_token: the "
                    "same steps replayed as one CUDA graph; both stream ~3.85 GB of weights per token "
                    "(2 layers + the 128256-row LM head), held as 16-bit hi + lo parts split once at load; "
                    "the GEMMs split only the activations"}


def glue_section(torch, heal, synthetic, dev, stream, reps):
    """The split kernel on the prefill weights and each decoder glue kernel on the decoder's
    prefill shapes (512 tokens, hidden 4096, 32/8 heads of 128, FFN 14336, vocab 128256),
    each timed with CUDA events over `reps` launches: a profiling case for the small kernels."""
    from error_compensated_gemm_b200.decoder import rope_tables
    n, H, Hq, Hkv, D, F, V = 512, 4096, 32, 8, 128, 14336, 128256
    W = synthetic.normal((4096, 14336), seed=1, std=0.02).to(dev)
    hi = torch.empty(W.shape, dtype=torch.int16, device=dev)
    lo = torch.empty_like(hi)
    table = synthetic.normal((V, H), seed=10).to(dev)
    ids = synthetic.prompt_ids(n, V).to(dev)
    h = torch.empty(n, H, device=dev)
    x = torch.empty(n, H, device=dev)
    qkv = synthetic.normal((n, (Hq + 2 * Hkv) * D), seed=11).to(dev)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    cos, sin = (t.to(dev) for t in rope_tables(1024, D, 500000.0))
    gu = synthetic.normal((n, 2 * F), seed=12).to(dev)
    act = torch.empty(n, F, device=dev)
    logits = synthetic.normal((8, V), seed=13).to(dev)
    am = torch.empty(8, dtype=torch.int32, device=dev)
    heads = synthetic.normal((1, Hq, n, D), seed=14).to(dev)
    rows = torch.empty(1, n, Hq, D, device=dev)
    calls = {
        "split_4096x14336": lambda: heal.heal_split(W, hi, lo),
        "embedding_gather": lambda: heal.heal_embedding_gather(table, ids, h),
        "rmsnorm": lambda: heal.heal_rmsnorm(h, None, x, 1e-5),
        "rope_q": lambda: heal.heal_rope(qkv, Hq, D, pos, cos, sin),
        "swiglu": lambda: heal.heal_swiglu(gu, act),
        "add": lambda: heal.heal_add(h, x),
        "argmax_8x128256": lambda: heal.heal_argmax(logits, am),
        "heads_to_rows": lambda: heal.heal_heads_to_rows(heads, rows),
    }
    out = {}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = {"us_per_launch": 1e3 * e0.elapsed_time(e1) / reps}
    st = heal.heal_get_device_status()
    if st != heal.HEAL_OK:
        raise SystemExit(f"device status: {heal.status_string(st)}")
    return out


# causal INT16 self-attention over a long prompt (the prefill kernel: 128-row query tiles on
# the tcgen05 tensor cores), timed in its own loop after the step
PREFILL_ATTN = {"B": 1, "T": 8192, "Hkv": 8, "Hq": 32, "D": 128}


def prefill_attention_section(torch, heal, synthetic, dev, stream, cap_stream, reps, peaks):
    c = PREFILL_ATTN
    B, T, Hkv, Hq, D = c["B"], c["T"], c["Hkv"], c["Hq"], c["D"]
    Qb, Kb, Vb = synthetic.kv_decode(B=B, T=T, Hkv=Hkv, Hq=Hq, D=D, Tq=T, seeds=(12, 13, 14))
    i16, f32 = torch.int16, torch.float32
    qc = torch.empty(B, Hq, T, D, dtype=i16, device=dev)
    qs = torch.empty(B, Hq, T, dtype=f32, device=dev)
    kc = torch.empty(B, Hkv, T, D, dtype=i16, device=dev)
    ks = torch.empty(B, Hkv, T, dtype=f32, device=dev)
    vc = torch.empty(B, Hkv, T, D, dtype=i16, device=dev)
    vs = torch.empty(B, Hkv, T, dtype=f32, device=dev)
    heal.heal_kv_quantize_int16(Qb.to(dev), qc, qs)
    heal.heal_kv_quantize_int16(Kb.to(dev), kc, ks)
    heal.heal_kv_quantize_int16(Vb.to(dev), vc, vs)
    kv_len = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, T, D, device=dev)
    aws = torch.empty(heal.heal_attention_workspace_bytes_gqa(B, Hq, Hkv, T, T), dtype=torch.uint8, device=dev)
    call = lambda: heal.heal_attention_int16(qc, qs, kc, ks, vc, vs, kv_len, D ** -0.5, out, aws, causal=True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap_stream):
        call()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    st = heal.heal_get_device_status()
    if st != heal.HEAL_OK:
        raise SystemExit(f"device status after prefill attention warm-up: {heal.status_string(st)}")
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(reps):
        g.replay()
    p1.record(stream)
    torch.cuda.synchronize()
    t = p0.elapsed_time(p1) / 1e3 / reps
    del g
    pairs = B * Hq * T * (T + 1) / 2                     # visible (query, token) pairs
    flop_eff = 4.0 * D * pairs                           # QK^T and PV, 2 flops per multiply-add
    i8_ops = 4 * 2.0 * D * pairs                         # four 8-bit integer products (S_hh, S_x x2, S_ll)
    f16_ops = 4 * 2.0 * D * pairs                        # four FP16 products (P_hi, r) x (256 V_hi, V_lo)
    peak16 = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    ideal = i8_ops / (2 * peak16 * 1e12) + f16_ops / (peak16 * 1e12)
    return {"config": dict(c, causal=True, Tq=T), "ms": 1e3 * t, "replays": reps,
            "tflops_effective": flop_eff / t / 1e12,
            "tensor_ops_per_s": (i8_ops + f16_ops) / t / 1e12,
            "roofline": {"bound": "tensor", "ideal_ms": 1e3 * ideal, "frac": ideal / t,
                         "peak": "bf16_tflops burst for the FP16 products, twice it for the 8-bit products"},
            "note": "conversion pass + tcgen05 attention kernel per call; timed separately after the step"}


def cpu_baseline_oracle(rows=4096):
    """The oracle's compensated GEMM (split + three FP64 products) on the prefill workload,
    restricted to `rows` rows of X; returns (TFLOP/s effective, seconds, threads)."""
    import numpy as np
    import synthetic
    from oracle import gemm as G
    M, K, N = PREFILL
    X, W = synthetic.gemm_prefill(M=M, K=K, N=N)
    Xs = X.numpy()[:rows]
    Wn = W.numpy()
    t0 = time.perf_counter()
    G.gemm_emulated(Xs, Wn)
    dt = time.perf_counter() - t0
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        threads = max((i.get("num_threads", 0) for i in info), default=threads) or threads
    except Exception:
        pass
    return 2.0 * rows * N * K / dt / 1e12, dt, threads


def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        # bind this rank's GPU before NCCL starts, so the barrier and the max-over-ranks
        # run on it
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


def arm_config(n):
    """The workload description both arms report (the same config for ours and the reference)."""
    M, K, N = PREFILL
    return {"workload": f"prefill linear X[{M}x{K}] (1% columns x20) . W[{K}x{N}], FP32, "
                        "in-kernel FP16 hi/lo split; step also runs decode GEMMs M=1/8/64 "
                        "(K=N=4096), the INT16 KV writer and INT16 decode attention "
                        "(B=8, 32q/8kv heads, D=128, context 8192)",
            "parallelism": f"independent shards x{n}" if n > 1 else "single GPU",
            "l2": "cold: before every part of a step, outside its events, a 256 MB buffer is written "
                  "and two other 256 MB buffers read (the part starts with none of its inputs in L2, no "
                  "dirty line of another part and the flush's own write-backs drained); part order: KV writer, prefill, attention, decode GEMMs, then two "
                  "torch streaming references (a 67 MB copy and a 67 MB read; not this library's kernels)"}


def reference_arm(args):
    ws, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return 0
    import numpy as np
    import synthetic
    from oracle import gemm as G
    M, K, N = PREFILL
    rows = 256
    X, W = synthetic.gemm_prefill(M=M, K=K, N=N)
    Xs, Wn = X.numpy()[:rows], W.numpy()
    for _ in range(args.warmup):
        G.gemm_emulated(Xs, Wn)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        G.gemm_emulated(Xs, Wn)
    dt = time.perf_counter() - t0
    val = 2.0 * rows * N * K * args.steps / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(args.gpus),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{rows} of {M} rows of X per step (FP64 split + three FP64 products "
                                   "of the prefill GEMM; the oracle, not tuned)"},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["prefill", "decode", "kv_writer", "attention", "attention_prefill", "glue"],
                    help="profiling case: run only this part of the step (glue: the split kernel and the "
                         "decoder glue kernels on the decoder's shapes)")
    ap.add_argument("--prefill-shape", default=None, help="M,N,K of the prefill GEMM (profiling case)")
    ap.add_argument("--kv-batch", type=int, default=None, help="batch of the KV workload (profiling case)")
    ap.add_argument("--prompt-len", type=int, default=None,
                    help="prompt length of the prefill attention workload (profiling case)")
    ap.add_argument("--no-decoder", action="store_true", help="skip the 2-layer decoder measurement")
    ap.add_argument("--no-study", action="store_true", help="skip the reproducibility analogue")
    ap.add_argument("--study", action="store_true",
                    help="reproducibility analogue: FP64 / FP32 / plain BF16 / HEAL pipelines on the decoder")
    args = ap.parse_args()
    if args.prefill_shape:
        global PREFILL
        PREFILL = tuple(int(v) for v in args.prefill_shape.split(","))
    if args.kv_batch:
        KV["B"] = args.kv_batch
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    import error_compensated_gemm_b200 as heal
    import synthetic
    from error_compensated_gemm_b200.shard import max_over_ranks
    ws, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    heal.lib()
    if args.study:
        from error_compensated_gemm_b200.study import reproducibility_study
        if rank == 0:
            print(json.dumps(reproducibility_study(dev)), flush=True)
        return 0
    peaks, peak_src = load_peaks()
    if args.only == "glue":
        res = glue_section(torch, heal, synthetic, dev, torch.cuda.current_stream(), max(1, args.steps))
        if rank == 0:
            print(json.dumps({"profiling_case": args.only, "result": res}), flush=True)
        return 0
    if args.only == "attention_prefill":
        if args.prompt_len:
            PREFILL_ATTN["T"] = args.prompt_len
        res = prefill_attention_section(torch, heal, synthetic, dev, torch.cuda.current_stream(),
                                        torch.cuda.Stream(), max(1, args.steps), peaks)
        if rank == 0:
            print(json.dumps({"profiling_case": args.only, "result": res}), flush=True)
        return 0
    wl = Workload(torch, heal, synthetic, dev, seed_offset=1000 * rank, only=args.only)
    for _ in range(max(3, args.warmup)):
        wl.run()
    torch.cuda.synchronize()
    cap_stream = torch.cuda.Stream()
    wl.capture(cap_stream)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        wl.run_graphs()
    torch.cuda.synchronize()
    st = heal.heal_get_device_status()
    if st != heal.HEAL_OK:
        raise SystemExit(f"device status after warm-up: {heal.status_string(st)}")

    dec_names = ([f"decode{m}" for m in DECODE_M] + [f"decode{m}_presplit" for m in DECODE_M] +
                 [f"decode{m}_w16" for m in DECODE_M] +
                 ["decode1_chain", "decode1_chain_presplit", "decode1_chain_w16", "ref_copy_67MB", "ref_read_67MB"])
    names = ["prefill"] + dec_names + ["kv_writer", "attention"]
    if args.only:
        keep = {"prefill": ["prefill"], "decode": dec_names,
                "kv_writer": ["kv_writer"], "attention": ["kv_writer", "attention"]}[args.only]
        names = keep
    evs = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in names}
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    smi_index = local
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    if vis:
        try:
            smi_index = int(vis.split(",")[local])
        except (ValueError, IndexError):
            smi_index = local
    with ClockSampler(smi_index) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            wl.run_graphs(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    st = heal.heal_get_device_status()
    if st != heal.HEAL_OK:
        raise SystemExit(f"device status after timing: {heal.status_string(st)}")
    total_ms = t_start.elapsed_time(t_end)
    part_ms = {n: sum(e[n][0].elapsed_time(e[n][1]) for e in evs) for n in names}
    if ws > 1:
        vals = max_over_ranks([total_ms] + [part_ms[n] for n in names], device=dev)
        total_ms = vals[0]
        part_ms = {n: vals[1 + i] for i, n in enumerate(names)}

    u = Workload.units()
    K = args.steps
    if args.only:
        if rank == 0:
            print(json.dumps({"profiling_case": args.only, "steps": K,
                              "ms_per_launch": {n: part_ms[n] / K for n in names},
                              "prefill_shape": PREFILL, "kv": KV}), flush=True)
        return 0
    prefill_s = part_ms["prefill"] / 1e3 / K          # per launch
    value = ws * u["prefill_flop_eff"] / prefill_s / 1e12
    mma_tflops = u["prefill_flop_mma"] / prefill_s / 1e12
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # The tensor denominator follows the clock the timed region ran at: the burst peak (a
    # short GEMM at full clock) unless the SM clock sampled under load fell well below its
    # maximum (power capping, as in the sustained measurement), then the sustained one.
    ck = clk.summary()
    at_max = bool(ck.get("sm_mhz") and ck.get("sm_max_mhz") and ck["sm_mhz"] >= 0.9 * ck["sm_max_mhz"])
    peak_tc, peak_tc_name = (peak_burst, "bf16_tflops (burst)") if at_max or not ck.get("sm_mhz") \
        else (peak_sus, "bf16_tflops_sustained")
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    attn_gbs = u["attn_bytes"] / (part_ms["attention"] / 1e3 / K) / 1e9
    kvw_gbs = u["kv_writer_bytes"] / (part_ms["kv_writer"] / 1e3 / K) / 1e9
    dec = {}
    for m in DECODE_M:
        for suffix, key in (("", f"M{m}"), ("_presplit", f"M{m}_presplit_weights")):
            t = part_ms[f"decode{m}{suffix}"] / 1e3 / K
            dec[key] = {"gbs": u["decode_bytes"][m] / t / 1e9, "us": 1e6 * t,
                        "frac_hbm": u["decode_bytes"][m] / t / 1e9 / hbm}
    for m in DECODE_M:
        t = part_ms[f"decode{m}_w16"] / 1e3 / K
        dec[f"M{m}_fp16_weights_two_products"] = {"gbs": u["decode16_bytes"][m] / t / 1e9, "us": 1e6 * t,
                                                  "frac_hbm": u["decode16_bytes"][m] / t / 1e9 / hbm}
    t = part_ms["ref_read_67MB"] / 1e3 / K
    dec["streaming_read_reference"] = {
        "us": 1e6 * t, "gbs": REF_COPY_BYTES / t / 1e9, "frac_hbm": REF_COPY_BYTES / t / 1e9 / hbm,
        "note": "torch one-dimensional sum over 67 MB (a decode GEMM's weight bytes, read once), timed in the step "
                "like the decode parts"}
    t = part_ms["ref_copy_67MB"] / 1e3 / K
    dec["streaming_copy_reference"] = {
        "us": 1e6 * t, "gbs": REF_COPY_BYTES / t / 1e9, "frac_hbm": REF_COPY_BYTES / t / 1e9 / hbm,
        "note": "torch device copy, 32 MB read + 32 MB written (a decode GEMM's weight bytes), timed in the step "
                "like the decode parts: what one launch of this size streams at"}
    for suffix, key, nb in (("", "M1_chain", "chain_bytes"), ("_presplit", "M1_chain_presplit_weights", "chain_bytes"),
                            ("_w16", "M1_chain_fp16_weights_two_products", "chain16_bytes")):
        t = part_ms[f"decode1_chain{suffix}"] / 1e3 / K
        dec[key] = {"gemms": CHAIN, "us_per_gemm": 1e6 * t / CHAIN, "gbs": u[nb] / t / 1e9,
                    "frac_hbm": u[nb] / t / 1e9 / hbm}

    # the prefill product with W split once into hi/lo beforehand (static weights), timed in
    # its own loop after the step so that it does not change the step's power and clocks
    presplit = splitpass = w16 = None
    if args.only is None and hasattr(wl, "Whi"):
        def time_call(fn):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                fn()
            for _ in range(3):
                g.replay()
            reps = max(10, min(K, 50))
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            with ClockSampler(smi_index) as cs:
                p0.record(stream)
                for _ in range(reps):
                    g.replay()
                p1.record(stream)
                torch.cuda.synchronize()
            t = p0.elapsed_time(p1) / 1e3 / reps
            if ws > 1:
                t = max_over_ranks([t], device=dev)[0]
            del g
            return t, reps, cs.summary()

        def pct_at_clock(flop_mma, t, ckx):
            """% of the 16-bit peak that applies at the clock sampled during this loop (a
            back-to-back GEMM loop can run into the power cap, unlike the mixed step)."""
            full = bool(ckx.get("sm_mhz") and ckx.get("sm_max_mhz") and ckx["sm_mhz"] >= 0.9 * ckx["sm_max_mhz"])
            pk = peak_burst if full or not ckx.get("sm_mhz") else peak_sus
            return 100.0 * flop_mma / t / 1e12 / pk, ("bf16_tflops (burst)" if pk == peak_burst else
                                                    "bf16_tflops_sustained")
        t_pre, reps, ck_pre = time_call(lambda: heal.heal_gemm_compensated(wl.X, wl.Whi, wl.C, b_lo=wl.Wlo))
        pc, pn = pct_at_clock(u["prefill_flop_mma"], t_pre, ck_pre)
        presplit = {"tflops_effective": ws * u["prefill_flop_eff"] / t_pre / 1e12,
                    "pct_of_16bit_peak": pc, "peak": pn, "clocks": ck_pre,
                    "ms": 1e3 * t_pre, "replays": reps,
                    "note": "the same product with W split once into hi/lo beforehand (static weights); "
                            "timed separately after the step"}
        t_sp, reps, ck_sp = time_call(lambda: heal.heal_gemm_compensated(wl.X, wl.W, wl.C, workspace=wl.wsp,
                                                                          b_split_pass=True))
        t_16, reps16, ck_16 = time_call(lambda: heal.heal_gemm_compensated(wl.X, wl.W16, wl.C, b_16bit=True))
        pc16, pn16 = pct_at_clock((2.0 / 3.0) * u["prefill_flop_mma"], t_16, ck_16)
        w16 = {"tflops_effective": ws * u["prefill_flop_eff"] / t_16 / 1e12,
               "pct_of_16bit_peak": pc16, "peak": pn16, "clocks": ck_16,
               "ms": 1e3 * t_16, "replays": reps16,
               "note": "the two-product form with FP16 weights (only X split; 2 MMAs); timed separately "
                       "after the step"}
        pcs, pns = pct_at_clock(u["prefill_flop_mma"], t_sp, ck_sp)
        splitpass = {"tflops_effective": ws * u["prefill_flop_eff"] / t_sp / 1e12,
                     "pct_of_16bit_peak": pcs, "peak": pns, "clocks": ck_sp,
                     "ms": 1e3 * t_sp, "replays": reps,
                     "note": "the same product with B split by a streaming pass into a workspace first "
                             "(b_split_pass; B's parts go through HBM); timed separately after the step"}

    attn_prefill = None
    if args.only is None:
        try:
            attn_prefill = prefill_attention_section(torch, heal, synthetic, dev, stream, cap_stream,
                                                     max(5, min(K, 20)), peaks)
        except SystemExit:
            raise
        except Exception as exc:  # report, do not hide
            attn_prefill = {"error": repr(exc)}
        if ws > 1:   # every rank takes this collective, failed or not
            mx = max_over_ranks([attn_prefill.get("ms", -1.0)], device=dev)[0]
            if "ms" in attn_prefill:
                attn_prefill["ms"] = mx

    # end to end through the public API: pinned host inputs -> device -> GEMM -> host result,
    # every step copying its inputs in and its result out.  Steps are pipelined the way a
    # caller streaming data would run them: two device buffer sets, the host-to-device copy
    # of step i+1 and the device-to-host copy of step i-1 on their own streams while step i
    # computes (PCIe carries both directions at once).
    M_, K_, N_ = PREFILL
    e2e = None
    try:
        hX = wl.X.cpu().pin_memory()
        hW = wl.W.cpu().pin_memory()
        hC = torch.empty(M_, N_, pin_memory=True)
        sets = [(torch.empty_like(wl.X), torch.empty_like(wl.W), torch.empty_like(wl.C)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_mm = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            k = i % 2
            dX, dW, dC = sets[k]
            if i >= 2:
                s_in.wait_event(ev_mm[k])        # step i-2's product has read this set's inputs
            with torch.cuda.stream(s_in):
                dX.copy_(hX, non_blocking=True)
                dW.copy_(hW, non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])     # step i-2's result has reached the host
            heal.heal_gemm_compensated(dX, dW, dC)
            ev_mm[k].record(stream)
            s_out.wait_event(ev_mm[k])
            with torch.cuda.stream(s_out):
                hC.copy_(dC, non_blocking=True)
                ev_out[k].record(s_out)

        reps = max(4, min(args.steps, 8))
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        for i in range(2, 2 + reps):
            e2e_step(i)
        stream.wait_event(ev_out[(1 + reps) % 2])   # the last step's result is on the host
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_s = e0.elapsed_time(e1) / 1e3 / reps
        if ws > 1:
            e2e_s = max_over_ranks([e2e_s], device=dev)[0]
        e2e = {"value": ws * u["prefill_flop_eff"] / e2e_s / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(4 * (M_ * K_ + K_ * N_)), "d2h_bytes_per_step": int(4 * M_ * N_),
               "note": "prefill GEMM through the library call with host buffers; copies of consecutive "
                       "steps overlap the product on separate streams (two device buffer sets)"}
        del sets
    except Exception as exc:  # report, do not hide
        e2e = {"error": repr(exc)}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tf, secs, thr = cpu_baseline_oracle()
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": f"full prefill workload (4096 rows), one run of FP64 split + three FP64 products, {secs:.1f} s"}

    dec_res = None
    if not args.no_decoder:
        dec_res = decoder_section(torch, heal, synthetic, dev, stream)
        if ws > 1:
            dec_res["prefill_ms"], dec_res["decode_ms_per_token"] = max_over_ranks(
                [dec_res["prefill_ms"], dec_res["decode_ms_per_token"]], device=dev)

    # the reproducibility analogue and the FP32-pipeline baseline (rank 0, after the timing)
    study = None
    if rank == 0 and not args.no_study:
        try:
            from error_compensated_gemm_b200.study import reproducibility_study
            study = reproducibility_study(dev)
        except Exception as exc:  # report, do not hide
            study = {"error": repr(exc)}

    # DRAM bytes of one prefill launch from the committed ncu summary (a full-size capture)
    traffic = None
    prof = os.path.join(ROOT, "profiles", "heal_gemm_pair_kernel_prefill_traffic.md")
    if os.path.exists(prof) and PREFILL == (4096, 4096, 14336):
        for ln in open(prof):
            if ln.startswith("bytes_per_launch:"):
                traffic = int(ln.split(":")[1])

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
            "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16x2-from-f32 (FP32 in/out, FP16 hi/lo tensor-core products, FP32 accumulate)",
            "data": "synthetic",
            "config": arm_config(ws),
            "pct_of_16bit_peak": 100.0 * mma_tflops / peak_tc,
            "prefill_presplit_weights": presplit,
            "prefill_split_pass_over_b": splitpass,
            "prefill_fp16_weights_two_products": w16,
            "attention_prefill": attn_prefill,
            "roofline": {"bound": "tensor", "achieved": mma_tflops, "peak": peak_tc, "unit": "TFLOP/s",
                         "frac": mma_tflops / peak_tc, "traffic": traffic,
                         "kernel": "heal_gemm_pair_kernel<1, 0, 0> (256x256 CTA pair, both operands split by the "
                                   "producer-side split warps)",
                         "peak_source": f"{peak_tc_name}, {peak_src}; chosen by the SM clock sampled under load "
                                        f"({ck.get('sm_mhz')} of {ck.get('sm_max_mhz')} MHz)",
                         "frac_of_burst_peak": mma_tflops / peak_burst,
                         "frac_of_sustained_peak": mma_tflops / peak_sus},
            "attn_gbs": attn_gbs, "attn_frac_hbm": attn_gbs / hbm,
            "secondary": {"kv_writer_gbs": kvw_gbs, "kv_writer_frac_hbm": kvw_gbs / hbm, "decode_gemm": dec,
                          "ms_per_step_parts": {n: part_ms[n] / K for n in names},
                          "hbm_peak_gbs": hbm, "peak_source": peak_src},
            "decoder": dec_res,
            "study": study,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": Workload.LAUNCHES_PER_STEP * K,
            "clocks": ck,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
