"""Benchmark of the spatial-temporal attention hot path on B200.

One step = one pass of every hot-path step of one attention block over one
batch of seeded synthetic inputs.  ``--workload`` picks the block:

* ``image_4096px`` (default): image-DiT full attention, B=1, N=65536 tokens
  (256x256 patches), 24 heads x 128, bf16, per-head RMSNorm on Q/K, KV in
  R=8 ring chunks merged by log-sum-exp, virtual Ulysses P=8 (ImageStep):
  SEQ2HEAD of V, K, Q (RMSNorm fused), attention, HEAD2SEQ of the output.
* ``vmajor_2304px``: V-Major selective attention, N=20736 (144x144), 24 x
  128 (VMajorStep): L1 change mask of V, compaction, cache update of the
  active tokens' K/V rows, attention of the fresh Q on the caches.
* ``opensora_low`` / ``video_1080p`` / ``tiny``: ST-DiT block (Step),
  B=1, T frames of S tokens, virtual P, N_T/N_S slices, R KV chunks:
  1. V-Major on the sending side: the L1 change of V against the previous
     step's V is measured on the spatially sharded layout, and only the
     active tokens take part in the all-to-all S->T -- their V rows and
     their per-head RMS-normalised K rows go straight into the K/V caches in
     the temporally sharded layout (vmajor_relayout_mask, which also writes
     the mask and the ascending list of active tokens, and
     vmajor_relayout_rows); ``--vmajor receiver`` moves all of K and V
     (ulysses_relayout), takes the mask there and scatters the active rows
     (vmajor_mask_compact, vmajor_scatter_rows) instead;
  2. all-to-all S->T of Q with the fused per-head RMSNorm (ulysses_relayout);
  3. spatial attention of the fresh Q against the cached K/V in R KV chunks
     and their log-sum-exp merge: by default all R chunks in one launch
     (st_attn_ring: each query block from its own chunk, the running
     statistics carried across the chunks); ``--attn chunks``, ``--merge
     separate`` or ``--schedule overlap`` take the chain instead: chunk 0
     writes the fp32 partial and its LSE (st_attn_spatial), every later chunk
     merges into it inside the attention kernel and the last one writes the
     result (st_attn_spatial_merge), or with ``--merge separate`` writes R
     partials merged by attn_chunk_merge;
  4. all-to-all T->S of the spatial output;
  5. temporal attention over the T frames of every token, read in place from
     the spatially sharded slice layout (st_attn_temporal).

value = attention FLOP of the step (4*rows*keys*D per head) / device time of
the step; the per-kernel breakdown (TFLOP/s or GB/s) is in "kernels".  Inputs
are resident in HBM; L2 is flushed (a 256 MiB write) between timed steps,
outside the timed events.  Under torchrun every rank runs its own replica
(weak scaling, no collective on the data path); the time is the max over
ranks.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "attention TFLOP/s & relayout GB/s on 1 B200, as fraction of bf16/HBM peak"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LAUNCHES_PER_STEP_BASE = 9            # receiver side: relayouts 3+1, vmajor 3 (mask, compaction, scatter),
                                      # merge 1, temporal 1; + R spatial launches; the fused merge has no
                                      # merge launch; sender side: mask + V rows, compaction and K rows
                                      # replace the K and V relayouts and the three vmajor launches (2 fewer)
SPATIAL_SRC = os.path.join(ROOT, "sequence_parallelism_st_b200", "csrc", "attn_spatial_sm100.cu")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK, "fallback"


def kernel_traffic(workload, launch):
    """DRAM bytes per launch of the roofline's attention launch from the
    committed ncu record (profiles/traffic.json: one entry per workload and
    launch kind), or None when the kernel source changed since the capture or
    nothing was captured for this workload."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = hashlib.sha256(open(SPATIAL_SRC, "rb").read()).hexdigest()[:16]
    for e in d.get("attn_fwd_sm100", []):
        if e.get("source_sha") == h and e.get("workload") == workload and e.get("launch") == launch:
            return e.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index, period=0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.stop_ev, self.thread, self.index = period, threading.Event(), None, index
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self.stop_ev.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *a):
        self.stop_ev.set()
        if self.thread:
            self.thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------- our arm
class Step:
    """Buffers and launches of one ST-DiT attention block step (all on one stream)."""

    def __init__(self, st, w, dev):
        self.st, self.w, self.dev = st, w, dev
        B, T, S, H, D, C, P = w.B, w.T, w.S, w.H, w.D, w.C, w.P
        n = B * T * S
        q, k, v = synth.qkv(w)                                # logical [B,T,S,H,D]
        vcur, vprev = synth.vmajor_pair(w, n, C)              # logical token order (b, t, s)
        self.tau = json.load(open(os.path.join(ROOT, "tests", "golden", "vmajor_tau.json")))[
            "workloads"][w.name]["0.5"]["tau"]
        self.n = n
        # the block's V is the V-Major "current" V; x layout holds shard p of every frame
        v = vcur.reshape(B, T, S, H, D)
        self.host = {"q": self.to_x(q), "k": self.to_x(k), "v": self.to_x(v)}
        self.gamma = synth.rms_gamma(w).to(dev)
        # previous step's V (in both layouts: the sender-side V-Major compares on x)
        # and the K/V caches, already in the temporally sharded (y) layout
        vprev_x = self.to_x(vprev.reshape(B, T, S, H, D))
        self.vprev_x = vprev_x.to(dev)
        vprev_y = self.x_to_y_host(vprev_x)
        kprev = synth.randn(w, "kprev", (B, T, S, H, D))
        kprev_y = self.x_to_y_host(self.to_x(kprev))
        self.d = {name: t.to(dev) for name, t in self.host.items()}
        self.vprev_y = vprev_y.to(dev)
        self.kcache0, self.vcache0 = kprev_y.to(dev), vprev_y.to(dev)
        self.kc, self.vc = self.kcache0.clone(), self.vcache0.clone()
        self.dt = st.ST_F32 if w.dtype == "f32" else st.ST_BF16       # the workload's element type
        mk = lambda dt=w.torch_dtype: torch.empty(n * C, dtype=dt, device=dev)
        self.qy, self.ky, self.vy, self.oy, self.ox, self.ot = mk(), mk(), mk(), mk(), mk(), mk()
        self.parts = [torch.empty(n * C, dtype=torch.float32, device=dev) for _ in range(w.R)]
        self.lses = [torch.empty(n * H, dtype=torch.float32, device=dev) for _ in range(w.R)]
        self.mask = torch.empty(n, dtype=torch.uint8, device=dev)
        self.idx = torch.empty(n, dtype=torch.int32, device=dev)
        self.count = torch.empty(1, dtype=torch.int32, device=dev)
        self.ws = torch.empty(max(16, st.vmajor_workspace_bytes(n)), dtype=torch.uint8, device=dev)
        # y layout with T/(N_T P) = 1: frames (q, i) of S contiguous tokens -> dense [1, T, S, H, D]
        assert T % (w.n_t * P) == 0 and T // (w.n_t * P) == 1
        self.sdesc = [st.make_desc(1, T, S, H, D, self.dt, kv_begin=c * S // w.R, kv_end=(c + 1) * S // w.R,
                                   o_fp32=1) for c in range(w.R)]
        # sender-side V-Major: the mask is taken on x and only active K/V rows move
        # (into the caches); receiver side: full relayouts, mask on y, scatter
        self.sender_vmajor = True
        # rotary position embedding of Q and K after their RMSNorm (positions: the
        # token index in the frame); off unless asked for
        self.rope_table = None
        # fused merge: chunk c >= 1 is merged into the accumulated fp32 partial
        # inside the attention kernel; the last chunk writes the bf16 result
        self.fused_merge = True
        # ring: the R chunks in one launch (each query block from its own
        # chunk, the running statistics carried across chunks, no partial)
        self.ring = False
        self.rdesc = st.make_desc(1, T, S, H, D, self.dt)
        self.sdesc_last = st.make_desc(1, T, S, H, D, self.dt, kv_begin=(w.R - 1) * S // w.R, kv_end=S,
                                       o_fp32=0)
        Tb, Sb = T // w.n_t, S // (w.n_s * P)
        self.tdesc = st.make_desc(P * B, T, S // P, H, D, self.dt, stride_b=w.n_t * w.n_s * Tb * Sb * C,
                                  stride_t=Sb * C, stride_s=C, t_block=Tb, stride_tb=w.n_s * Tb * Sb * C,
                                  s_block=Sb, stride_sb=Tb * Sb * C)
        # per-kernel timing events (launching stream = torch's current stream)
        self.ev = {}

    def to_x(self, t):
        """Logical [B,T,S,H,D] -> stacked x shards [P,B,N_T,N_S,T/N_T,S/(N_S P),C]."""
        w = self.w
        X = t.reshape(w.B, w.T, w.S, w.C)
        Tb, Sb = w.T // w.n_t, w.S // (w.n_s * w.P)
        return X.reshape(w.B, w.n_t, Tb, w.n_s, w.P, Sb, w.C).permute(4, 0, 1, 3, 2, 5, 6).contiguous().reshape(-1)

    def x_to_y_host(self, x):
        """Host-side layout change used only to prepare the previous step's buffers."""
        w = self.w
        Tb, Sb = w.T // w.n_t, w.S // (w.n_s * w.P)
        X = x.reshape(w.P, w.B, w.n_t, w.n_s, Tb, Sb, w.C).permute(1, 2, 4, 3, 0, 5, 6)  # b i t1 j p s1 c
        X = X.reshape(w.B, w.T, w.S, w.C)        # logical
        Tq, Ss = w.T // (w.n_t * w.P), w.S // w.n_s
        Y = X.reshape(w.B, w.n_t, w.P, Tq, w.n_s, Ss, w.C).permute(2, 0, 1, 4, 3, 5, 6)
        return Y.contiguous().reshape(-1)

    def reset_caches(self):
        self.kc.copy_(self.kcache0)
        self.vc.copy_(self.vcache0)

    def _mark(self, name, start):
        if self.timing:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            self.ev.setdefault(name, []).append(e) if start else self.ev[name].append(e)

    def run(self, timing=False):
        st, w, d = self.st, self.w, self.d
        self.timing = timing
        P, B, T, S, C, D = w.P, w.B, w.T, w.S, w.C, w.D
        if self.sender_vmajor:
            # V-Major on the sending side: V's change decides which tokens take
            # part in the exchange; their V and (normalised) K rows go straight
            # into the caches, Q moves whole
            self._mark("vmajor", True)
            st.vmajor_relayout_mask(d["v"], self.vprev_x, self.vc, P, B, T, S, C, w.n_t, w.n_s, self.tau, self.mask,
                                    self.idx, self.count, self.ws)
            st.vmajor_relayout_rows(d["k"], self.kc, self.idx, self.count, P, B, T, S, C, w.n_t, w.n_s,
                                    rms_gamma=self.gamma, rms_head_dim=D, rms_eps=w.rms_eps,
                                    rope_table=self.rope_table)
            self._mark("vmajor", False)
            self._mark("relayout_s2t", True)
            self._qk_relayout(d["q"], self.qy)
            self._mark("relayout_s2t", False)
        else:
            # V first: its exchange needs no normalisation ([CC] "V-First")
            self._mark("relayout_s2t", True)
            st.ulysses_relayout("S2T", d["v"], self.vy, P, B, T, S, C, w.n_t, w.n_s)
            self._qk_relayout(d["k"], self.ky)
            self._qk_relayout(d["q"], self.qy)
            self._mark("relayout_s2t", False)
            self._mark("vmajor", True)
            st.vmajor_mask_compact(self.vy.view(self.n, C), self.vprev_y.view(self.n, C), self.tau, self.mask,
                                   self.idx, self.count, self.ws)
            st.vmajor_scatter_rows(self.idx, self.count, [self.ky.view(self.n, C), self.vy.view(self.n, C)],
                                   [self.kc.view(self.n, C), self.vc.view(self.n, C)])
            self._mark("vmajor", False)
        if self.ring:
            self._mark("spatial", True)
            st.st_attn_ring(self.qy, self.kc, self.vc, self.oy, self.lses[0], w.R, desc=self.rdesc)
            self._mark("spatial", False)
        elif self.fused_merge:
            self._spatial_fused(None)
        else:
            self._mark("spatial", True)
            for c in range(w.R):
                st.st_attn_spatial(self.qy, self.kc, self.vc, self.parts[c], self.lses[c], desc=self.sdesc[c])
            self._mark("spatial", False)
            self._mark("merge", True)
            st.attn_chunk_merge(self.parts, self.lses, B * T, S, w.H, D, self.oy)
            self._mark("merge", False)
        self._mark("relayout_t2s", True)
        st.ulysses_relayout("T2S", self.oy, self.ox, P, B, T, S, C, w.n_t, w.n_s)
        self._mark("relayout_t2s", False)
        self._mark("temporal", True)
        st.st_attn_temporal(d["q"], d["k"], d["v"], self.ot, None, desc=self.tdesc)
        self._mark("temporal", False)

    def _qk_relayout(self, src, dst):
        """S->T of Q or K with the per-head RMSNorm (and the rotary embedding when on)."""
        st, w = self.st, self.w
        if self.rope_table is not None:
            st.ulysses_relayout_rope("S2T", src, dst, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, rms_gamma=self.gamma,
                                     rms_head_dim=w.D, rms_eps=w.rms_eps, rope_table=self.rope_table)
        else:
            st.ulysses_relayout("S2T", src, dst, w.P, w.B, w.T, w.S, w.C, w.n_t, w.n_s, rms_gamma=self.gamma,
                                rms_head_dim=w.D, rms_eps=w.rms_eps)

    def _spatial_fused(self, i):
        """KV chunks of the spatial attention with the merge fused into the
        kernel: chunk 0 writes the fp32 partial and its LSE, chunks 1..R-2 merge
        into it in place, chunk R-1 merges and writes the bf16 result (and the
        merged LSE).  i: shard range of the overlapped schedule, or None."""
        st, w = self.st, self.w
        descs = self.sdesc if i is None else self.sdesc_sl[i]
        last = self.sdesc_last if i is None else self.sdesc_last_sl[i]
        self._mark("spatial", True)
        st.st_attn_spatial(self.qy, self.kc, self.vc, self.parts[0], self.lses[0], desc=descs[0])
        self._mark("spatial", False)
        self._mark("spatial_merge", True)
        for c in range(1, w.R - 1):
            st.st_attn_spatial_merge(self.qy, self.kc, self.vc, self.parts[0], self.lses[0], self.parts[0],
                                     self.lses[0], desc=descs[c])
        st.st_attn_spatial_merge(self.qy, self.kc, self.vc, self.parts[0], self.lses[0], self.oy, self.lses[1],
                                 desc=last)
        self._mark("spatial_merge", False)

    # ------------------------------------------------------------ overlapped schedule
    def setup_overlap(self, n_slices, att_sms):
        """Buffers and streams of the chunk-and-overlap schedule: the step is cut
        into n_slices ranges of temporally sharded shards; the attention of one
        range runs on att_sms SMs (high-priority stream) while the memory-bound
        steps of the neighbouring ranges run on the others (low-priority stream)."""
        w = self.w
        assert w.P % n_slices == 0
        self.n_sl, self.att_sms = n_slices, att_sms
        self.sender_vmajor = False          # the shard-range schedule moves whole ranges (receiver side)
        self.s_att = torch.cuda.Stream(priority=-8)     # mapped to the highest priority the device has
        self.s_mem = torch.cuda.Stream(priority=0)
        n_sl_tok = self.n // n_slices
        self.counts = torch.zeros(n_slices, dtype=torch.int32, device=self.dev)
        T = w.T
        self.sdesc_sl = [[self.st.make_desc(1, T, w.S, w.H, w.D, self.dt, kv_begin=c * w.S // w.R,
                                            kv_end=(c + 1) * w.S // w.R, o_fp32=1, n_slices=n_slices, slice=i)
                          for c in range(w.R)] for i in range(n_slices)]
        self.sdesc_last_sl = [self.st.make_desc(1, T, w.S, w.H, w.D, self.dt,
                                                kv_begin=(w.R - 1) * w.S // w.R, kv_end=w.S, o_fp32=0,
                                                n_slices=n_slices, slice=i) for i in range(n_slices)]
        self.n_sl_tok = n_sl_tok

    def _prep(self, i):
        """S->T relayout of shard range i and the V-Major steps of its tokens."""
        st, w, d = self.st, self.w, self.d
        P, B, T, S, C, D = w.P, w.B, w.T, w.S, w.C, w.D
        per = P // self.n_sl
        sh = (i * per, (i + 1) * per)
        st.ulysses_relayout_range("S2T", d["v"], self.vy, P, B, T, S, C, w.n_t, w.n_s, shards=sh)
        st.ulysses_relayout_range("S2T", d["k"], self.ky, P, B, T, S, C, w.n_t, w.n_s, shards=sh,
                                  rms_gamma=self.gamma, rms_head_dim=D, rms_eps=w.rms_eps)
        st.ulysses_relayout_range("S2T", d["q"], self.qy, P, B, T, S, C, w.n_t, w.n_s, shards=sh,
                                  rms_gamma=self.gamma, rms_head_dim=D, rms_eps=w.rms_eps)
        t0, t1 = i * self.n_sl_tok, (i + 1) * self.n_sl_tok
        rows = lambda t: t.view(self.n, C)[t0:t1]
        cnt = self.counts[i:i + 1]
        st.vmajor_mask_compact(rows(self.vy), rows(self.vprev_y), self.tau, self.mask[t0:t1],
                               self.idx[t0:t1], cnt, self.ws)
        st.vmajor_scatter_rows(self.idx[t0:t1], cnt, [rows(self.ky), rows(self.vy)], [rows(self.kc), rows(self.vc)])

    def _post(self, i):
        """Merge of the KV-chunk partials of shard range i and its T->S relayout."""
        st, w = self.st, self.w
        P, B, T, S, C, D, H = w.P, w.B, w.T, w.S, w.C, w.D, w.H
        per = P // self.n_sl
        f0, f1 = i * T // self.n_sl, (i + 1) * T // self.n_sl
        e0, e1 = f0 * S * C, f1 * S * C
        l0, l1 = f0 * H * S, f1 * H * S
        if not self.fused_merge:
            st.attn_chunk_merge([p[e0:e1] for p in self.parts], [x[l0:l1] for x in self.lses], B * (f1 - f0), S, H,
                                D, self.oy[e0:e1])
        st.ulysses_relayout_range("T2S", self.oy, self.ox, P, B, T, S, C, w.n_t, w.n_s, shards=(i * per, (i + 1) * per))

    def run_overlap(self):
        """One step on the overlapped schedule; ordered after, and followed by,
        the current stream's work."""
        st, w, d = self.st, self.w, self.d
        main = torch.cuda.current_stream()
        n_sl, mem_sms = self.n_sl, self.st_num_sms() - self.att_sms
        start = torch.cuda.Event()
        start.record(main)
        self.s_att.wait_event(start)
        self.s_mem.wait_event(start)
        e_prep = [torch.cuda.Event() for _ in range(n_sl)]
        e_att = [torch.cuda.Event() for _ in range(n_sl)]
        e_go = [torch.cuda.Event() for _ in range(n_sl)]
        try:
            with torch.cuda.stream(self.s_mem):
                st.st_set_sm_budget(0)                  # nothing else runs yet
                self._prep(0)
                e_prep[0].record(self.s_mem)
            for i in range(n_sl):
                with torch.cuda.stream(self.s_att):
                    self.s_att.wait_event(e_prep[i])
                    e_go[i].record(self.s_att)          # attention of range i may start
                    st.st_set_sm_budget(self.att_sms)
                    if self.fused_merge:
                        self._spatial_fused(i)
                    else:
                        for c in range(w.R):
                            st.st_attn_spatial(self.qy, self.kc, self.vc, self.parts[c], self.lses[c],
                                               desc=self.sdesc_sl[i][c])
                    e_att[i].record(self.s_att)
                with torch.cuda.stream(self.s_mem):
                    self.s_mem.wait_event(e_go[i])      # let the attention take its SMs first
                    st.st_set_sm_budget(mem_sms)
                    if i + 1 < n_sl:
                        self._prep(i + 1)
                        e_prep[i + 1].record(self.s_mem)
                    if i == 0:
                        st.st_attn_temporal(d["q"], d["k"], d["v"], self.ot, None, desc=self.tdesc)
                    if i >= 1:
                        self.s_mem.wait_event(e_att[i - 1])
                        self._post(i - 1)
            with torch.cuda.stream(self.s_mem):
                self.s_mem.wait_event(e_att[n_sl - 1])
                st.st_set_sm_budget(0)
                self._post(n_sl - 1)
        finally:
            st.st_set_sm_budget(0)
        main.wait_stream(self.s_mem)
        main.wait_stream(self.s_att)

    def st_num_sms(self):
        return torch.cuda.get_device_properties(self.dev).multi_processor_count

    def kernel_times(self):
        out = {}
        for name, evs in self.ev.items():
            ts = [evs[i].elapsed_time(evs[i + 1]) for i in range(0, len(evs) - 1, 2)]
            out[name] = sum(ts) / len(ts)
        return out

    # ------------------------------------------------------------ bench interface
    def outputs(self):
        """Device results a caller reads back after the step."""
        return [self.ox, self.ot]

    def set_io(self, d, outs):
        self.d = d
        self.ox, self.ot = outs

    def flops(self):
        return self.w.spatial_flops() + self.w.temporal_flops()

    def active_tokens(self):
        return int(self.count.item()) if not hasattr(self, "n_sl") else int(self.counts.sum().item())

    def launches(self):
        w = self.w
        if hasattr(self, "n_sl"):
            return (3 + 3 + w.R + (1 if self.fused_merge else 2)) * self.n_sl + 1
        # sender-side V-Major: V mask-relayout, compaction and K rows (3) replace 2 relayouts + 3 V-Major launches
        spatial = 1 if self.ring else w.R - (1 if self.fused_merge else 0)
        return LAUNCHES_PER_STEP_BASE + spatial - (2 if self.sender_vmajor else 0)

    def group_flops(self):
        """Attention FLOP of each timed kernel group (the tensor-bound ones)."""
        w, R = self.w, self.w.R
        sp = w.spatial_flops()
        if self.ring:
            return {"spatial": sp, "temporal": w.temporal_flops()}
        if self.fused_merge:
            return {"spatial": sp / R, "spatial_merge": sp * (R - 1) / R, "temporal": w.temporal_flops()}
        return {"spatial": sp, "temporal": w.temporal_flops()}

    def group_bytes(self, frac_active):
        return kernel_bytes(self.w, frac_active, self.sender_vmajor)

    def roofline_name(self):
        return "ring" if self.ring else "chunk0"

    def roofline_launch(self, ktimes):
        """(flop of one launch of the dominant kernel, its mean duration in ms):
        the ring launch, or the chunk-0 spatial launch of the chunk chain."""
        w = self.w
        if self.ring:
            return w.spatial_flops(), ktimes["spatial"]
        return w.spatial_flops() / w.R, ktimes["spatial"] / (1 if self.fused_merge else w.R)

    def describe(self, args):
        w = self.w
        return {"B": w.B, "T": w.T, "S": w.S, "H": w.H, "D": w.D, "P": w.P, "N_T": w.n_t, "N_S": w.n_s,
                "kv_chunks": w.R,
                "schedule": "serial" if not hasattr(self, "n_sl") else
                f"overlap: {self.n_sl} shard ranges, attention on {self.att_sms} SMs",
                "chunk_merge": ("one launch, stationary chunk first, running (m, l, O) carried across chunks"
                                if self.ring else "fused into the attention kernel" if self.fused_merge
                                else "attn_chunk_merge"),
                "vmajor": "sender side (mask on x, active K/V rows into the caches)" if self.sender_vmajor else
                "receiver side (full relayouts, mask on y, scatter)",
                "qk_rope": self.rope_table is not None}


class ImageStep:
    """Buffers and launches of one image-DiT full-attention block step: B = 1,
    N tokens of H heads x D, virtual Ulysses partition P, R KV ring chunks.

      1. SEQ2HEAD of V (V first: it needs no normalisation), then of K and Q
         with the per-head RMSNorm fused into the move (ulysses_relayout);
         the head-sharded layout [P, B, H/P, N, D] holds each head's sequence
         contiguously, so its B*H head sequences are the attention's frames;
      2. full attention over the N keys in R ring chunks merged by log-sum-exp:
         ``ring`` runs one launch that walks each query block's chunks from its
         own (stationary) chunk onwards and carries the running max, row sum and
         O across the chunk boundaries (st_attn_ring); ``chunks`` runs chunk 0
         (st_attn_spatial, fp32 partial + LSE) and merges every later chunk
         into it inside the attention kernel (st_attn_spatial_merge);
      3. HEAD2SEQ of the output back to the sequence-sharded layout.
    """

    def __init__(self, st, w, dev, attn="ring"):
        self.st, self.w, self.dev, self.attn = st, w, dev, attn
        N, H, D, C, P, B = w.S, w.H, w.D, w.C, w.P, w.B
        assert w.T == 1 and N % P == 0 and H % P == 0
        q, k, v = synth.qkv(w)                                # [B, 1, N, H, D] = the stacked sequence shards
        self.host = {"q": q.reshape(-1), "k": k.reshape(-1), "v": v.reshape(-1)}
        self.d = {name: t.to(dev) for name, t in self.host.items()}
        self.gamma = synth.rms_gamma(w).to(dev)
        mk = lambda dt=torch.bfloat16: torch.empty(B * N * C, dtype=dt, device=dev)
        self.qy, self.ky, self.vy, self.oy, self.ox = mk(), mk(), mk(), mk(), mk()
        self.lse = [torch.empty(B * H * N, dtype=torch.float32, device=dev) for _ in range(2)]
        R = w.R
        # head-sharded y: frames (p, b, h1) of N contiguous tokens, one head each
        self.frames = B * H
        if attn == "ring":
            self.rdesc = st.make_desc(1, self.frames, N, 1, D, st.ST_BF16)
        else:
            self.part = mk(torch.float32)
            self.sdesc = [st.make_desc(1, self.frames, N, 1, D, st.ST_BF16, kv_begin=c * N // R,
                                       kv_end=(c + 1) * N // R, o_fp32=0 if c == R - 1 else 1) for c in range(R)]
        self.ev = {}
        self.timing = False

    _mark = Step._mark
    kernel_times = Step.kernel_times

    def run(self, timing=False):
        st, w, d = self.st, self.w, self.d
        self.timing = timing
        P, B, N, H, D = w.P, w.B, w.S, w.H, w.D
        self._mark("relayout_seq2head", True)
        st.ulysses_relayout("SEQ2HEAD", d["v"], self.vy, P, B, N, H, D)
        st.ulysses_relayout("SEQ2HEAD", d["k"], self.ky, P, B, N, H, D, rms_gamma=self.gamma, rms_head_dim=D,
                            rms_eps=w.rms_eps)
        st.ulysses_relayout("SEQ2HEAD", d["q"], self.qy, P, B, N, H, D, rms_gamma=self.gamma, rms_head_dim=D,
                            rms_eps=w.rms_eps)
        self._mark("relayout_seq2head", False)
        self._mark("spatial", True)
        if self.attn == "ring":
            st.st_attn_ring(self.qy, self.ky, self.vy, self.oy, self.lse[0], w.R, desc=self.rdesc)
            self._mark("spatial", False)
        elif w.R == 1:
            st.st_attn_spatial(self.qy, self.ky, self.vy, self.oy, self.lse[0], desc=self.sdesc[0])
            self._mark("spatial", False)
        else:
            st.st_attn_spatial(self.qy, self.ky, self.vy, self.part, self.lse[0], desc=self.sdesc[0])
            self._mark("spatial", False)
            self._mark("spatial_merge", True)
            for c in range(1, w.R - 1):
                st.st_attn_spatial_merge(self.qy, self.ky, self.vy, self.part, self.lse[0], self.part, self.lse[0],
                                         desc=self.sdesc[c])
            st.st_attn_spatial_merge(self.qy, self.ky, self.vy, self.part, self.lse[0], self.oy, self.lse[1],
                                     desc=self.sdesc[w.R - 1])
            self._mark("spatial_merge", False)
        self._mark("relayout_head2seq", True)
        st.ulysses_relayout("HEAD2SEQ", self.oy, self.ox, P, B, N, H, D)
        self._mark("relayout_head2seq", False)

    def outputs(self):
        return [self.ox]

    def set_io(self, d, outs):
        self.d = d
        (self.ox,) = outs

    def flops(self):
        return self.w.spatial_flops()

    def active_tokens(self):
        return None

    def launches(self):
        return 3 + (1 if self.attn == "ring" else self.w.R) + 1

    def group_flops(self):
        sp, R = self.w.spatial_flops(), self.w.R
        if self.attn == "ring" or R == 1:
            return {"spatial": sp}
        return {"spatial": sp / R, "spatial_merge": sp * (R - 1) / R}

    def group_bytes(self, frac_active):
        t = self.w.tensor_bytes()
        return {"relayout_seq2head": 3 * 2 * t, "relayout_head2seq": 2 * t}

    def roofline_name(self):
        return "ring" if self.attn == "ring" else "chunk0"

    def roofline_launch(self, ktimes):
        """The ring launch (all R chunks), or the chunk-0 launch of the chunk chain."""
        sp = self.w.spatial_flops()
        return (sp if self.attn == "ring" else sp / self.w.R), ktimes["spatial"]

    def describe(self, args):
        w = self.w
        return {"B": w.B, "N": w.S, "H": w.H, "D": w.D, "P": w.P, "kv_chunks": w.R, "qk_rmsnorm": True,
                "relayout": "SEQ2HEAD (V, then K and Q with the RMSNorm) -> attention -> HEAD2SEQ",
                "chunk_merge": ("one launch, stationary chunk first, running (m, l, O) carried across chunks"
                                if self.attn == "ring" else
                                "chunk 0 partial, later chunks merged inside the attention kernel")}


class VMajorStep:
    """Buffers and launches of one V-Major selective attention step: N tokens of
    H heads x D (T = 1), fresh Q, K and V of this step, the previous step's V
    and the K/V caches.

      1. per-token L1 change of V against the previous step's V, the mask
         (L1 > tau), the ascending list of active tokens and the update of the
         K/V caches with the active tokens' rows (vmajor_mask_compact_scatter);
      2. attention of the fresh Q against the cached K/V (st_attn_spatial).
    tau is the golden threshold for the active fraction f.
    """

    def __init__(self, st, w, dev, frac=0.5):
        self.st, self.w, self.dev = st, w, dev
        N, H, D, C = w.S, w.H, w.D, w.C
        assert w.B == 1 and w.T == 1
        self.n = N
        q = synth.randn(w, "q", (1, 1, N, H, D))
        cur_v, prev_v = synth.vmajor_pair(w, N, C)
        cur_k, prev_k = synth.vmajor_pair(w, N, C, prev="kprev", noise="knoise")
        self.frac_target = frac
        self.tau = json.load(open(os.path.join(ROOT, "tests", "golden", "vmajor_tau.json")))[
            "workloads"][w.name][str(frac)]["tau"]
        self.host = {"q": q.reshape(-1), "k": cur_k.reshape(-1), "v": cur_v.reshape(-1)}
        self.d = {name: t.to(dev) for name, t in self.host.items()}
        self.vprev = prev_v.reshape(-1).to(dev)
        self.kcache0, self.vcache0 = prev_k.reshape(-1).to(dev), prev_v.reshape(-1).to(dev)
        self.kc, self.vc = self.kcache0.clone(), self.vcache0.clone()
        self.o = torch.empty(N * C, dtype=torch.bfloat16, device=dev)
        self.mask = torch.empty(N, dtype=torch.uint8, device=dev)
        self.idx = torch.empty(N, dtype=torch.int32, device=dev)
        self.count = torch.empty(1, dtype=torch.int32, device=dev)
        self.ws = torch.empty(max(16, st.vmajor_workspace_bytes(N)), dtype=torch.uint8, device=dev)
        self.desc = st.make_desc(1, 1, N, H, D, st.ST_BF16)
        self.ev = {}
        self.timing = False

    _mark = Step._mark
    kernel_times = Step.kernel_times

    def reset_caches(self):
        self.kc.copy_(self.kcache0)
        self.vc.copy_(self.vcache0)

    def run(self, timing=False):
        st, d, n, C = self.st, self.d, self.n, self.w.C
        self.timing = timing
        self._mark("vmajor", True)
        st.vmajor_mask_compact_scatter(d["v"].view(n, C), self.vprev.view(n, C), self.tau, self.mask, self.idx,
                                       self.count, self.ws, [d["k"].view(n, C), d["v"].view(n, C)],
                                       [self.kc.view(n, C), self.vc.view(n, C)])
        self._mark("vmajor", False)
        self._mark("spatial", True)
        st.st_attn_spatial(d["q"], self.kc, self.vc, self.o, None, desc=self.desc)
        self._mark("spatial", False)

    def outputs(self):
        return [self.o]

    def set_io(self, d, outs):
        self.d = d
        (self.o,) = outs

    def flops(self):
        return self.w.spatial_flops()

    def active_tokens(self):
        return int(self.count.item())

    def launches(self):
        return 3                      # mask with the fused cache update, compaction, attention

    def group_flops(self):
        return {"spatial": self.w.spatial_flops()}

    def group_bytes(self, frac_active):
        # the least traffic of the work: V and its previous value read, the
        # active rows of K read, the active rows of K and V written into the caches
        t = self.w.tensor_bytes()
        return {"vmajor": 2 * t + 3 * frac_active * t}

    def roofline_name(self):
        return "cached_kv"

    def roofline_launch(self, ktimes):
        return self.w.spatial_flops(), ktimes["spatial"]

    def describe(self, args):
        w = self.w
        return {"B": w.B, "N": w.S, "H": w.H, "D": w.D, "vmajor_target_fraction": self.frac_target,
                "vmajor": "mask + compaction + cache update of active K/V rows, attention on the caches"}


STEPS = {"st": Step, "image": ImageStep, "vmajor": VMajorStep}


def step_kind(w):
    """The step a workload runs: image-DiT full attention (T = 1 with the Q/K
    RMSNorm), V-Major selective attention (T = 1 with change fractions), or the
    ST-DiT block."""
    if w.T == 1 and w.vmajor_f and not w.rms:
        return "vmajor"
    if w.T == 1:
        return "image"
    return "st"


def kernel_bytes(w, frac_active, sender=False):
    """Algorithmic HBM bytes per step of each memory-bound kernel group."""
    e = w.elem_bytes
    t = w.B * w.T * w.S * w.C * e               # one [B,T,S,C] tensor
    if sender:
        # V and its previous value read once on x, the active rows of V written
        # and of K read and written; Q moved whole
        return {"relayout_s2t": 2 * t, "vmajor": 2 * t + 3 * frac_active * t,
                "merge": w.R * (2 * t + w.B * w.T * w.S * w.H * 4) + t, "relayout_t2s": 2 * t, "temporal": 4 * t}
    return {
        "relayout_s2t": 3 * 2 * t,
        "merge": w.R * (2 * t + w.B * w.T * w.S * w.H * 4) + t,  # fp32 partials + LSE in, bf16 out
        "vmajor": 2 * t + 2 * 2 * frac_active * t,
        "relayout_t2s": 2 * t,
        "temporal": 4 * t,
    }


def max_over_ranks(total_ms, world, dev):
    """The job's time: the largest of the ranks' device times (every rank
    takes part in the same collective; a single rank returns its own)."""
    if world <= 1:
        return float(total_ms)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, flop_per_replica_step, ms_per_step):
    """Whole-job throughput in TFLOP/s: every rank runs one replica of the step
    (weak scaling), so the job does world x the flop of a step per step time."""
    return world * flop_per_replica_step / (ms_per_step * 1e-3) / 1e12


def make_step(st, args, w, dev):
    kind = step_kind(w)
    if kind == "image":
        return ImageStep(st, w, dev, attn="chunks" if args.attn == "chunks" else "ring")
    if kind == "vmajor":
        return VMajorStep(st, w, dev, frac=args.vmajor_f)
    stp = Step(st, w, dev)
    stp.fused_merge = args.merge == "fused"
    stp.ring = args.attn == "ring" and args.merge == "fused" and args.schedule == "serial"
    stp.sender_vmajor = args.vmajor == "sender"
    if args.rope:
        stp.rope_table = st.st_rope_table(w.S, w.D, 10000.0, device=dev)
    if args.schedule == "overlap":
        stp.setup_overlap(args.slices, args.att_sms)
    return stp


def run_ours(args, w, rank, world, dev):
    import sequence_parallelism_st_b200 as st
    stp = make_step(st, args, w, dev)
    step_fn = stp.run_overlap if hasattr(stp, "n_sl") else stp.run
    launches = stp.launches()
    pk, pk_src = peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step_fn()
    torch.cuda.synchronize()
    if st.st_check_device_status() != st.ST_OK:
        raise RuntimeError("device status not OK after warm-up")
    active = stp.active_tokens()
    # ---- timed: device time of exactly K steps, L2 flushed between steps outside the events
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                      else int(os.environ.get("LOCAL_RANK", 0))) as clk:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record()
            step_fn()
            ends[i].record()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    status = st.st_check_device_status()
    # per-kernel breakdown from a separate pass: events between the kernel
    # groups would otherwise sit inside the timed steps
    for _ in range(max(3, args.steps // 4)):
        flush.zero_()
        stp.run(timing=True)
    torch.cuda.synchronize()
    ktimes = stp.kernel_times()
    # ---- end to end through the C ABI with host buffers: H2D of the step's inputs,
    #      the step, D2H of its outputs, all inside the events
    pinned_in = {k: v.pin_memory() for k, v in stp.host.items()}
    h2d = sum(v.numel() * v.element_size() for v in pinned_in.values())
    # Pipelined across steps: step i's inputs go up on one copy stream while
    # step i-1 computes and step i-2's results come down on another, with
    # two device sets of inputs and outputs.  Every step still carries its
    # own host->device and device->host copies inside the timed region.
    outs0 = stp.outputs()
    d_sets = [stp.d, {k: torch.empty_like(v) for k, v in stp.d.items()}]
    o_sets = [outs0, [torch.empty_like(o) for o in outs0]]
    out_host = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs0] for _ in range(2)]
    d2h = sum(v.numel() * v.element_size() for v in out_host[0])
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_pass(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(comp)
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])      # set j's inputs no longer read
                for k2, v2 in pinned_in.items():
                    d_sets[j][k2].copy_(v2, non_blocking=True)
                ev_in[i].record(s_in)
            comp.wait_event(ev_in[i])
            if i >= 2:
                comp.wait_event(ev_out[i - 2])           # set j's outputs already copied down
            stp.set_io(d_sets[j], o_sets[j])
            step_fn()
            ev_comp[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                for hb, db in zip(out_host[j], o_sets[j]):
                    hb.copy_(db, non_blocking=True)
                ev_out[i].record(s_out)
        comp.wait_event(ev_out[n - 1])
        b.record(comp)
        b.synchronize()
        return a.elapsed_time(b) / n

    e2e_pass(3)                                          # warm-up of the pipeline
    n_e2e = max(4, args.steps // 4)
    e2e_ms = [e2e_pass(n_e2e)]
    stp.set_io(d_sets[0], o_sets[0])
    if rank != 0:
        return None
    f = stp.flops()
    n_steps = args.steps
    ms = total_ms / n_steps
    value = whole_job_value(world, f, ms)
    e2e_val = whole_job_value(world, f, statistics.mean(e2e_ms))
    frac_active = None if active is None else active / stp.n
    gb = stp.group_bytes(frac_active or 0.0)
    gf = stp.group_flops()
    kernels = {}
    for name, t in ktimes.items():
        ent = {"ms": round(t, 5)}
        if name in gf:
            ent["tflops"] = round(gf[name] / (t * 1e-3) / 1e12, 2)
            if name != "temporal":
                ent["frac_of_bf16_peak"] = round(ent["tflops"] / pk["bf16_tflops"], 4)
        if name in gb:
            ent["gbs"] = round(gb[name] / (t * 1e-3) / 1e9, 1)
            ent["frac_of_hbm_peak"] = round(ent["gbs"] / pk["hbm_gbs"], 4)
        kernels[name] = ent
    # roofline of the dominant kernel: the spatial / full attention launch.
    # Peak: the burst GEMM figure while the clocks ran free, the sustained one
    # when the power cap throttled them during the timed region.
    fl_launch, launch_ms = stp.roofline_launch(ktimes)
    achieved = fl_launch / (launch_ms * 1e-3) / 1e12
    clocks = clk.summary()
    capped = "sw_power_cap" in clocks.get("reasons", []) and "bf16_tflops_sustained" in pk
    tc_peak = pk["bf16_tflops_sustained"] if capped else pk["bf16_tflops"]
    tc_src = f"{pk_src} bf16 " + ("sustained (power cap active)" if capped else "burst")
    cfg = {"workload": w.name}
    cfg.update(stp.describe(args))
    cfg.update({"parallelism": f"replicas{world}",
                "l2": "flushed between timed steps (256 MiB write, outside the step events)"})
    if frac_active is not None:
        cfg["vmajor_active"] = round(frac_active, 4)
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": n_steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": cfg,
        "e2e": {"value": round(e2e_val, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(statistics.mean(e2e_ms), 5)},
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_sm100 (st_attn_*)", "achieved": round(achieved, 2),
                     "peak": tc_peak, "peak_source": tc_src, "unit": "TFLOP/s",
                     "frac": round(achieved / tc_peak, 4), "frac_of_burst": round(achieved / pk["bf16_tflops"], 4),
                     "traffic": kernel_traffic(w.name, stp.roofline_name()),
                     "algorithmic_flop_per_launch": fl_launch, "launch_ms": round(launch_ms, 5)},
        "kernels": kernels,
        "gpu_launches": launches * n_steps,
        "device_status": st.st_status_string(status),
        "clocks": clocks,
        "cpu_baseline": cpu_baseline(w, budget_s=args.cpu_budget) if world == 1 and args.cpu_budget > 0 else None,
    }


# ---------------------------------------------------------------- oracle arm
class OracleSample:
    """The fp64 oracle on a bounded sample of one step of workload ``w``.

    ST-DiT step: spatial attention of whole frames and temporal attention of a
    set of tokens.  Image step: the attention rows of a set of query tokens
    (every head, all N keys) on Q and K normalised by the oracle's RMSNorm.
    V-Major step: the attention rows of a set of query tokens against the K/V
    caches the oracle's mask, compaction and cache update produce.  The
    preparation (input generation, RMSNorm of the whole K, mask, cache update,
    fp64 conversion) happens before any timing; ``run`` times the sampled
    attention only.
    """

    def __init__(self, w):
        import numpy as np
        import oracle
        self.w, self.kind = w, step_kind(w)
        self.np, self.oracle = np, oracle
        if self.kind == "st":
            self.q, self.k, self.v = synth.qkv(w)
            return
        N, H, D, C = w.S, w.H, w.D, w.C
        shape = (1, 1, N, H, D)
        if self.kind == "image":
            q, k, v = synth.qkv(w)
            g = synth.rms_gamma(w)
            self.k = oracle.rmsnorm_heads(k.reshape(N, C), g, D, w.rms_eps).reshape(shape)
            self.q_raw, self.g = q.reshape(N, C), g
            self.v = v.to(torch.float64).numpy().reshape(shape)
        else:
            q = synth.randn(w, "q", shape)
            cur_v, prev_v = synth.vmajor_pair(w, N, C)
            cur_k, prev_k = synth.vmajor_pair(w, N, C, prev="kprev", noise="knoise")
            tau = json.load(open(os.path.join(ROOT, "tests", "golden", "vmajor_tau.json")))[
                "workloads"][w.name]["0.5"]["tau"]
            idx, cnt = oracle.compact(oracle.change_mask(oracle.l1_change(cur_v, prev_v), tau))
            self.k = oracle.scatter_rows(idx, cnt, cur_k, prev_k).reshape(shape)
            self.v = oracle.scatter_rows(idx, cnt, cur_v, prev_v).reshape(shape)
            self.q_raw = q.reshape(N, C)

    def unit_flop(self):
        """FLOP of one sampled unit: a frame (ST) or a query row (image, V-Major)."""
        w = self.w
        if self.kind == "st":
            return 4.0 * w.B * w.S * w.S * w.C
        return 4.0 * w.S * w.C

    def full_flop(self):
        w = self.w
        return w.spatial_flops() + (w.temporal_flops() if self.kind == "st" else 0.0)

    def run(self, n_units, n_tokens=0):
        """Times the oracle on n_units frames (ST, plus temporal attention of
        n_tokens tokens) or n_units query rows.  Returns (seconds, flop)."""
        np, oracle, w = self.np, self.oracle, self.w
        if self.kind == "st":
            t0 = time.perf_counter()
            oracle.spatial(self.q, self.k, self.v, frames=list(range(n_units)))
            if n_tokens:
                oracle.temporal(self.q, self.k, self.v, tokens=np.arange(n_tokens))
            dt = time.perf_counter() - t0
            return dt, n_units * self.unit_flop() + 4.0 * w.B * n_tokens * w.T * w.T * w.C
        N, H, D, C = w.S, w.H, w.D, w.C
        rows = np.arange(n_units) * max(1, N // max(n_units, 1)) % N
        t0 = time.perf_counter()
        for r0 in range(0, len(rows), 64):                   # 64 query rows per call bounds the score matrix
            sel = rows[r0:r0 + 64]
            q = self.q_raw[torch.from_numpy(sel)]
            if self.kind == "image":
                q = oracle.rmsnorm_heads(q, self.g, D, w.rms_eps)
            if isinstance(q, torch.Tensor):
                q = q.to(torch.float64).numpy()
            q = q.reshape(1, 1, len(sel), H, D)
            oracle.spatial(q, self.k, self.v, kv=(0, N))     # every query row attends to all N keys
        dt = time.perf_counter() - t0
        return dt, len(rows) * self.unit_flop()


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def _fit_units(sample, budget_s, cap, probe, n_tokens=0):
    """Units of the sample whose timing fills about budget_s seconds."""
    dt, _ = sample.run(probe, n_tokens)
    per = max(dt / probe, 1e-4)
    return max(1, min(cap, int(budget_s / per)))


def cpu_baseline(w, budget_s=15.0):
    """The oracle timed on the host cores on a bounded sample of the step (all
    cores, then one BLAS thread on a smaller sample), with the full-size step
    time extrapolated linearly from the per-unit time (every unit -- a frame or
    a query row -- costs the same)."""
    from threadpoolctl import threadpool_limits
    smp = OracleSample(w)
    st_kind = smp.kind == "st"
    cap = w.T if st_kind else w.S
    probe = 1 if st_kind else 64
    n_tok = min(1200, w.S) if st_kind else 0       # tokens of the temporal sample (a frame's worth at most)
    units = _fit_units(smp, budget_s, cap, probe, n_tok)
    dt, fl = smp.run(units, n_tok)
    val = fl / dt / 1e12
    full_s = smp.full_flop() / (val * 1e12)
    with threadpool_limits(limits=1):
        u1 = max(1, min(units, _fit_units(smp, budget_s / 3, cap, 1 if st_kind else 16)))
        dt1, fl1 = smp.run(u1, 0 if st_kind else 0)
    val1 = fl1 / dt1 / 1e12
    what = (f"spatial attention of {units} of {w.T} frames (all heads, all {w.S} queries and keys) + temporal "
            f"attention of {n_tok} of {w.S} tokens" if st_kind else
            f"attention rows of {units} of {w.S} query tokens (all {w.H} heads, all {w.S} keys)"
            + (" on RMS-normalised Q/K" if smp.kind == "image" else " on the oracle-updated K/V caches"))
    return {"value": round(val, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle: {what}; {dt:.1f} s",
            "single_thread": {"value": round(val1, 6), "unit": "TFLOP/s", "cores": 1,
                              "sample": f"{u1} {'frames' if st_kind else 'query rows'}, {dt1:.1f} s"},
            "extrapolated_full_step_s": {"all_cores": round(full_s, 1),
                                         "single_thread": round(smp.full_flop() / (val1 * 1e12), 1),
                                         "note": "extrapolated linearly from the sampled units"}}


def run_reference(args, w):
    smp = OracleSample(w)
    st_kind = smp.kind == "st"
    cap = w.T if st_kind else w.S
    n_tok = min(300, w.S) if st_kind else 0
    units = _fit_units(smp, args.cpu_budget / max(args.steps, 1), cap, 1 if st_kind else 16, n_tok)
    if not st_kind:
        units = max(8, units // 8 * 8)
    for _ in range(args.warmup):
        smp.run(1 if st_kind else 8, min(64, w.S) if st_kind else 0)
    times, fls = [], []
    for _ in range(args.steps):
        dt, fl = smp.run(units, n_tok)
        times.append(dt)
        fls.append(fl)
    tot = sum(times)
    val = sum(fls) / tot / 1e12
    ms = 1e3 * tot / args.steps
    if st_kind:
        sample = (f"fp64 numpy oracle per step: spatial attention of {units} of {w.T} frames (all heads, all "
                  f"{w.S} queries and keys) + temporal attention of {n_tok} of {w.S} tokens")
    else:
        sample = (f"fp64 numpy oracle per step: attention rows of {units} of {w.S} query tokens (all {w.H} heads, "
                  f"all {w.S} keys)")
    # n_gpus: the launch's N, so the line pairs with ours at the same N (the
    # oracle itself runs on rank 0's host cores, as cpu_baseline says)
    n_launch = int(os.environ.get("WORLD_SIZE", 1))
    return {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": n_launch,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "S": w.S, "H": w.H, "D": w.D},
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="image_4096px", choices=sorted(synth.BY_NAME))
    ap.add_argument("--attn", choices=["ring", "chunks"], default="ring",
                    help="ring = one launch over every KV chunk (each query block from its own chunk); "
                         "chunks = one launch per chunk, later chunks merged inside the attention kernel "
                         "(--merge separate: attn_chunk_merge)")
    ap.add_argument("--vmajor-f", type=float, default=0.5, choices=[0.1, 0.5, 0.9],
                    help="V-Major step: target active fraction of the golden threshold")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time for cpu_baseline (0: no cpu_baseline)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="image workload only: run it at this many tokens instead (profiler captures)")
    ap.add_argument("--merge", choices=["fused", "separate"], default="fused",
                    help="fused: KV chunks 1..R-1 merged inside the attention kernel; separate: attn_chunk_merge")
    ap.add_argument("--vmajor", choices=["sender", "receiver"], default="sender",
                    help="sender: mask on x, only active K/V rows move into the caches; receiver: full relayouts, "
                         "mask on y, scatter")
    ap.add_argument("--rope", action="store_true",
                    help="rotary position embedding of Q and K after their RMSNorm (token index in the frame)")
    ap.add_argument("--schedule", choices=["serial", "overlap"], default="serial",
                    help="overlap: shard ranges of the step on two streams (attention / memory-bound steps)")
    ap.add_argument("--slices", type=int, default=4, help="shard ranges of the overlap schedule")
    ap.add_argument("--att-sms", type=int, default=120, help="SMs of the attention stream in the overlap schedule")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = synth.BY_NAME[args.workload]
    if args.tokens:
        # a smaller instance of the image step (same kernels), for profiler captures
        if step_kind(w) != "image" or args.tokens % w.P:
            ap.error("--tokens applies to the image workload and must be a multiple of its P")
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}@N{args.tokens}", S=args.tokens)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        res = run_ours(args, w, rank, world, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
