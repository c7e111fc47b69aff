"""Benchmark of the DV-SSQ layer on B200: one JSON line on rank 0.

Default step (the Spark-shaped down_proj: W 2560 x 10240 BF16, H_256 blocks,
1280 salient columns, rank 16): encode W -> forward of 1 token -> forward of
16 tokens.  The unit is GB/s of algorithmic bytes: the encoder reads W once
and writes the packed form; each forward reads the packed layer once (x and y
are not counted).  Eight independent copies of the layer are used in
rotation so that no step finds its inputs in the 126 MB L2, and the forwards
of a step read a copy that was encoded four steps earlier.

Other workloads (--workload): decode (the two forwards only), prefill (4096
tokens through the up_proj, TFLOP/s), bulk_encode (all 108 matrices of the
36-layer Spark MLP stack) and stack (one token through the 36 x (gate, up,
GELU, down) stack, 1.9 GB of packed weights per token).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload spark_down|decode|prefill|bulk_encode|stack]

The timed region replays one CUDA graph per rotation slot (--no-graphs
launches eagerly instead).  With --gpus N > 1 (under torchrun, one process
per GPU) every rank runs the same step on its own layers: the path has no
data-path exchange, so scaling is weak and the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DV-SSQ linear fwd: decode HBM GB/s vs peak; prefill TFLOP/s; encode GB/s"
N_COPIES = 8
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------- helpers --

def packed_bytes(M, K, rank, n_sal):
    return M * K // 2 + M * (K // 64) * 2 + M * n_sal + M * 2 + n_sal * 4 + M * rank * 2 + rank * K * 2


def encode_bytes(M, K, n_sal):
    # read W once (BF16) + write q4, s4, q8, s8, sal_idx
    return M * K * 2 + M * K // 2 + M * (K // 64) * 2 + M * n_sal + M * 2 + n_sal * 4


def kernel_bytes(name, M, K, rank, n_sal, T):
    """Algorithmic bytes of one launch of each kernel (see the design notes).

    The decode GEMV (dec_row for one or two tokens, dec_main above) reads the
    packed layer except U; dec_tail reads U.  x, y and the partial sums are
    not counted."""
    if name == "enc_pass1":
        return M * K * 2
    if name == "enc_pass2":
        return encode_bytes(M, K, n_sal)
    if name in ("dec_row", "dec_main"):
        return packed_bytes(M, K, rank, n_sal) - M * rank * 2
    if name == "dec_tail":
        return M * rank * 2
    return None


# The source files each kernel is built from: a recorded DRAM count stays valid
# while these files are unchanged.
# Roofline bars of the task: the decode GEMV kernels at 0.70 of measured HBM,
# the prefill GEMM at 0.50 of the measured BF16 tensor peak.
ROOFLINE_TARGETS = {"dec_row": 0.70, "dec_main": 0.70, "mlp_stack": 0.70, "pre_gemm": 0.50}

KERNEL_SOURCES = {
    "enc_pass1": ("encode.cu", "fwht_group.cuh", "exact_sum.cuh"),
    "enc_pass2": ("encode.cu", "fwht_group.cuh", "exact_sum.cuh"),
    "enc_select": ("encode.cu",),
    "dec_row": ("decode_row.cu", "fwht_group.cuh"),
    "dec_main": ("decode.cu", "fwht_group.cuh"),
    "dec_tail": ("decode.cu",),
    "pre_act": ("prefill.cu", "fwht_group.cuh"),
    "pre_mat": ("prefill.cu",),
    "pre_gemm": ("prefill.cu", "common.cuh"),
    "mlp_stack": ("stack.cu", "common.cuh"),
    "materialize": ("materialize.cu",),
    "lr_mul": ("lowrank.cu",),
    "bss_logits": ("attention.cu",),
    "bss_pv": ("attention.cu",),
}


def _code_only(text):
    """Source text without // comments and blank lines: a comment edit does
    not change the kernel, so it must not invalidate a capture."""
    out = []
    for line in text.splitlines():
        q, cut = False, len(line)
        for i, ch in enumerate(line):
            if ch == '"' and (i == 0 or line[i - 1] != "\\"):
                q = not q
            elif not q and line.startswith("//", i):
                cut = i
                break
        line = line[:cut].rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def source_hash(kernel=None):
    d = os.path.join(ROOT, "mixed_precision_weight_b200", "csrc")
    files = KERNEL_SOURCES.get(kernel) or tuple(sorted(os.listdir(d)))
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update((f + _code_only(fh.read())).encode())
    return h.hexdigest()[:16]


def dram_traffic(kernel, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if still current."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except OSError:
        return None
    ent = rec.get(f"{kernel}@{workload}")
    if not ent or ent.get("source_hash") != source_hash(kernel):
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc = index, None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)   # let the sampler start before the timed region
        return self

    def __exit__(self, *a):
        self.out, self.err = "", ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, self.err = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, self.err = self.proc.communicate()
            if not self.out.strip():
                print(f"clock sampler produced no samples: {self.err.strip()[:300]}",
                      file=sys.stderr)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- workload --

class SparkDownStep:
    """encode + forward(T=1) + forward(T=16) on rotating copies of one layer."""

    name = "spark_down_proj_2560x10240_r16_encode+fwd_T1+T16"

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv, self.torch = dv, torch
        wl = synth.WORKLOADS["spark_down"]
        self.wl = wl
        M, K, B, r, n = wl.M, wl.K, wl.block, wl.rank, wl.n_sal
        self.M, self.K, self.r, self.n = M, K, r, n
        self.shape = dv.Shape.make(M, K, B, r, n)
        self.copies = []
        for c in range(N_COPIES):
            off = 100 * rank_id + c
            W = wl.weight(seed_offset=off).to(device)
            act = wl.act_scale(seed_offset=off).to(device)
            U, V = synth.lowrank_factors(M, K, r, seed=wl.seed + 7 + off)
            packed = dv.PackedWeights.empty(self.shape, device, U=U.to(device), V=V.to(device))
            self.copies.append((W, act, packed))
        self.x1 = wl.activations(1, seed_offset=rank_id).to(device)
        self.x16 = wl.activations(16, seed_offset=rank_id).to(device)
        self.ws_enc = torch.empty(dv.dvssq_encode_workspace_size(self.shape), dtype=torch.uint8,
                                  device=device)
        self.ws1 = torch.empty(dv.dvssq_forward_workspace_size(self.shape, 1), dtype=torch.uint8,
                               device=device)
        self.ws16 = torch.empty(dv.dvssq_forward_workspace_size(self.shape, 16), dtype=torch.uint8,
                                device=device)
        self.y1 = torch.empty((1, M), dtype=torch.float32, device=device)
        self.y16 = torch.empty((16, M), dtype=torch.float32, device=device)
        for c in range(N_COPIES):   # every copy starts encoded
            W, act, packed = self.copies[c]
            dv.dvssq_encode(self.shape, W, act, packed, workspace=self.ws_enc)
        self.i = 0

    graph_slots = N_COPIES

    def step_slot(self, i):
        dv = self.dv
        W, act, packed = self.copies[i % N_COPIES]
        dv.dvssq_encode(self.shape, W, act, packed, workspace=self.ws_enc)
        fwd = self.copies[(i + N_COPIES // 2) % N_COPIES][2]
        dv.dvssq_linear_forward(self.shape, fwd, self.x1, y=self.y1, workspace=self.ws1)
        dv.dvssq_linear_forward(self.shape, fwd, self.x16, y=self.y16, workspace=self.ws16)

    def step(self):
        self.step_slot(self.i)
        self.i += 1

    def bytes_per_step(self):
        return encode_bytes(self.M, self.K, self.n) + 2 * packed_bytes(self.M, self.K, self.r, self.n)

    def launches_per_step(self):
        return 3 + 2 + 2

    def config(self):
        return {"workload": self.name, "M": self.M, "K": self.K, "block": 256, "rank": self.r,
                "n_sal": self.n, "tokens": [1, 16],
                "step": "dvssq_encode + dvssq_linear_forward(T=1) + dvssq_linear_forward(T=16)",
                "l2": f"{N_COPIES} rotating layer copies (~{N_COPIES * 70} MB) > 126 MB L2; "
                      "forwards read a copy encoded 4 steps earlier",
                "lowrank_factors": "seeded synthetic U, V (values do not change the work)",
                "parallelism": "replica per GPU (weak scaling, no data-path collective)"}

    # ---- end-to-end through the public API with host buffers ----
    def e2e_setup(self, synth):
        torch = self.torch
        wl = self.wl
        self.hW = wl.weight(seed_offset=999).pin_memory()
        self.hact = wl.act_scale(seed_offset=999).pin_memory()
        U, V = synth.lowrank_factors(self.M, self.K, self.r, seed=1234)
        self.hU, self.hV = U.pin_memory(), V.pin_memory()
        self.hx1 = wl.activations(1, seed_offset=77).pin_memory()
        self.hx16 = wl.activations(16, seed_offset=78).pin_memory()
        self.hy1 = torch.empty((1, self.M), dtype=torch.float32).pin_memory()
        self.hy16 = torch.empty((16, self.M), dtype=torch.float32).pin_memory()

    def e2e_step(self):
        dv = self.dv
        layer = dv.DvssqLinear.from_weight(self.hW, self.hact, self.hU, self.hV, block=256)
        self.hy1.copy_(layer(self.hx1), non_blocking=True)
        self.hy16.copy_(layer(self.hx16), non_blocking=True)

    def e2e_bytes(self):
        h2d = sum(t.numel() * t.element_size() for t in
                  (self.hW, self.hact, self.hU, self.hV, self.hx1, self.hx16))
        d2h = (self.hy1.numel() + self.hy16.numel()) * 4
        return h2d, d2h

    # ---- the oracle on the host cores ----
    def oracle_sample(self, O, synth):
        wl = self.wl
        W = O.torch_bf16_to_f64(wl.weight(seed_offset=555))
        act = wl.act_scale(seed_offset=555).numpy()
        U, V = synth.lowrank_factors(self.M, self.K, self.r, seed=55)
        Uf, Vf = O.torch_bf16_to_f64(U), O.torch_bf16_to_f64(V)
        x1 = O.torch_bf16_to_f64(wl.activations(1))
        x16 = O.torch_bf16_to_f64(wl.activations(16))

        def step():
            enc = O.encode(W, act, wl.block, self.r, with_svd=False)
            O.forward(enc, x1, U=Uf, V=Vf)
            O.forward(enc, x16, U=Uf, V=Vf)
        return step


class DecodeStep(SparkDownStep):
    """forward(T=1) + forward(T=16) only, on rotating pre-encoded copies."""

    name = "spark_down_proj_2560x10240_r16_fwd_T1+T16"

    def step_slot(self, i):
        dv = self.dv
        fwd = self.copies[i % N_COPIES][2]
        dv.dvssq_linear_forward(self.shape, fwd, self.x1, y=self.y1, workspace=self.ws1)
        dv.dvssq_linear_forward(self.shape, fwd, self.x16, y=self.y16, workspace=self.ws16)

    def bytes_per_step(self):
        return 2 * packed_bytes(self.M, self.K, self.r, self.n)

    def launches_per_step(self):
        return 4

    def config(self):
        c = super().config()
        c.update(workload=self.name,
                 step="dvssq_linear_forward(T=1) + dvssq_linear_forward(T=16)",
                 l2=f"{N_COPIES} rotating encoded layers (~{N_COPIES * 18} MB) > 126 MB L2")
        return c

    def e2e_step(self):
        # tokens in from pinned host memory, outputs back to the host
        layer = self.dv.DvssqLinear(self.shape, self.copies[self.i % N_COPIES][2])
        self.hy1.copy_(layer(self.hx1), non_blocking=True)
        self.hy16.copy_(layer(self.hx16), non_blocking=True)
        self.i += 1

    def e2e_bytes(self):
        return ((self.hx1.numel() + self.hx16.numel()) * 2,
                (self.hy1.numel() + self.hy16.numel()) * 4)

    def oracle_sample(self, O, synth):
        wl = self.wl
        enc = O.encode(O.torch_bf16_to_f64(wl.weight(seed_offset=555)),
                       wl.act_scale(seed_offset=555).numpy(), wl.block, self.r, with_svd=False)
        U, V = synth.lowrank_factors(self.M, self.K, self.r, seed=55)
        Uf, Vf = O.torch_bf16_to_f64(U), O.torch_bf16_to_f64(V)
        x1 = O.torch_bf16_to_f64(wl.activations(1))
        x16 = O.torch_bf16_to_f64(wl.activations(16))

        def step():
            O.forward(enc, x1, U=Uf, V=Vf)
            O.forward(enc, x16, U=Uf, V=Vf)
        return step


class PrefillStep:
    """forward of 4096 tokens through the Spark up_proj layer (tensor cores)."""

    name = "spark_up_proj_10240x2560_r16_prefill_T4096"
    unit = "TFLOP/s"

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv, self.torch = dv, torch
        wl = synth.WORKLOADS["spark_up_prefill"]
        self.wl = wl
        self.M, self.K, self.r, self.n, self.T = wl.M, wl.K, wl.rank, wl.n_sal, 4096
        self.shape = dv.Shape.make(wl.M, wl.K, wl.block, wl.rank)
        U, V = synth.lowrank_factors(wl.M, wl.K, wl.rank, seed=wl.seed + rank_id)
        self.packed = dv.PackedWeights.empty(self.shape, device, U=U.to(device), V=V.to(device))
        dv.dvssq_encode(self.shape, wl.weight(seed_offset=rank_id).to(device),
                        wl.act_scale(seed_offset=rank_id).to(device), self.packed)
        self.x = wl.activations(self.T, seed_offset=rank_id).to(device)
        self.ws = torch.empty(dv.dvssq_forward_workspace_size(self.shape, self.T), dtype=torch.uint8,
                              device=device)
        self.y = torch.empty((self.T, self.M), dtype=torch.float32, device=device)

    graph_slots = 1

    def step_slot(self, i):
        self.dv.dvssq_linear_forward(self.shape, self.packed, self.x, y=self.y, workspace=self.ws)

    def step(self):
        self.step_slot(0)

    def work_per_step(self):
        return 2.0 * self.T * self.M * self.K + 2.0 * self.T * self.r * (self.K + self.M)

    def kernel_work(self, name):
        if name == "pre_gemm":
            return self.work_per_step()
        salp = (self.n + 63) // 64 * 64
        kc = self.K + salp + 64
        if name == "pre_act":
            # x read + Xc written
            return self.T * self.K * 2 + self.T * kc * 2
        if name == "pre_mat":
            # packed layer read + materialised A written
            return packed_bytes(self.M, self.K, self.r, self.n) + self.M * kc * 2
        return None

    def launches_per_step(self):
        return 2

    def config(self):
        return {"workload": self.name, "M": self.M, "K": self.K, "block": 256, "rank": self.r,
                "n_sal": self.n, "tokens": self.T,
                "step": "dvssq_linear_forward(T=4096) on tcgen05",
                "flops": "2*T*M*K + 2*T*r*(K+M) (algorithmic; the kernel also multiplies the "
                         "dense-layout zeros and the salient tier)",
                "l2": "x (21 MB) + packed layer (17.6 MB); each step reruns the same layer",
                "parallelism": "replica per GPU"}


class BulkEncodeStep:
    """encode of all 108 MLP matrices of the 36-layer Spark shape (one pass)."""

    name = "spark_mlp_36x3_bulk_encode"

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv, self.torch = dv, torch
        H, I = 2560, 10240
        # four BF16 sources per shape (4 x 3 x 52 MB > L2), used in rotation so
        # that every encode reads its matrix from HBM
        gen_cache = {}
        for which, (M, K) in enumerate(((I, H), (I, H), (H, I))):
            for c in range(4):
                W = synth.weight(M, K, seed=10 + which + 7 * c + 100 * rank_id,
                                 n_outlier_cols=max(1, K // 1000), outlier_scale=15.0).to(device)
                act = synth.act_scale(K, seed=20 + which + 7 * c).to(device)
                gen_cache[(which, c)] = (W, act)
        self.shapes = {w: dv.Shape.make(M, K, 256, 16) for w, (M, K) in
                       enumerate(((I, H), (I, H), (H, I)))}
        self.packed = {w: dv.PackedWeights.empty(self.shapes[w], device) for w in range(3)}
        self.src = gen_cache
        ws = max(dv.dvssq_encode_workspace_size(sh) for sh in self.shapes.values())
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.H, self.I = H, I

    def step(self):
        for layer in range(36):
            for w in range(3):
                W, act = self.src[(w, layer % 4)]
                self.dv.dvssq_encode(self.shapes[w], W, act, self.packed[w], workspace=self.ws)

    def bytes_per_step(self):
        H, I = self.H, self.I
        return 36 * (2 * encode_bytes(I, H, H // 8) + encode_bytes(H, I, I // 8))

    def launches_per_step(self):
        return 108 * 3

    def kernel_work(self, name):
        H, I = self.H, self.I
        per = {"enc_pass1": (2 * I * H * 2 + H * I * 2) / 3,
               "enc_pass2": (2 * encode_bytes(I, H, H // 8) + encode_bytes(H, I, I // 8)) / 3}
        return per.get(name)

    def config(self):
        return {"workload": self.name, "matrices": 108, "weights": 108 * 2560 * 10240,
                "step": "dvssq_encode of 36 x (gate, up, down)",
                "l2": "each matrix's BF16 source (52 MB) is read from HBM by pass 1; "
                      "pass 2 re-reads it, partly from L2",
                "parallelism": "replica per GPU"}


class StackStep:
    """One token through the 36-layer Spark MLP stack (decode, T = 1).

    Per layer: g = gate(x), u = up(x) (BF16 outputs), h = RN_bf16(gelu(g) u),
    x = down(h) (BF16); gate/up are 10240 x 2560 and down 2560 x 10240, rank
    16 (layers 0..13 and 29..35) or 24 (14..28).  The 108 packed matrices
    (1.9 GB) far exceed L2, so every token streams them all from HBM."""

    name = "spark_mlp_stack_36x(gate,up,down)_T1"
    graph_slots = 1
    n_layers = 36     # the full model; --layers sets fewer for profiling
    fused = True      # one cooperative launch per token (dvssq_mlp_stack_forward)

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv, self.torch, self.device = dv, torch, device
        H, I = 2560, 10240
        self.H, self.I = H, I
        self.layers = []
        ws = 0
        self.nl = self.n_layers
        for l in range(self.nl):
            r = synth.stack_rank(l)
            mats = []
            for which, (M, K) in enumerate(((I, H), (I, H), (H, I))):
                seed = synth.layer_seed(1 + rank_id, l, which)
                shape = dv.Shape.make(M, K, 256, r)
                W = synth.weight_device(M, K, seed, device, n_outlier_cols=max(1, K // 1000),
                                        outlier_scale=15.0)
                act = synth.act_scale(K, seed).to(device)
                U, V = synth.lowrank_factors(M, K, r, seed=seed + 17)
                packed = dv.PackedWeights.empty(shape, device, U=U.to(device), V=V.to(device))
                need = dv.dvssq_encode_workspace_size(shape)
                if need > ws:
                    self.ws_enc = torch.empty(need, dtype=torch.uint8, device=device)
                    ws = need
                dv.dvssq_encode(shape, W, act, packed, workspace=self.ws_enc)
                del W
                mats.append((shape, packed))
            self.layers.append(mats)
        del self.ws_enc
        fw = max(dv.dvssq_forward_workspace_size(sh, 1) for mats in self.layers for sh, _ in mats)
        self.ws = torch.empty(fw, dtype=torch.uint8, device=device)
        self.mstack = dv.MlpStack(self.layers, device=device) if self.fused else None
        self.x0 = synth.activations(1, H, seed=3 + rank_id, n_outlier=13,
                                    outlier_scale=25.0).to(device)
        self.x = torch.empty((1, H), dtype=torch.bfloat16, device=device)
        self.g = torch.empty((1, I), dtype=torch.bfloat16, device=device)
        self.u = torch.empty((1, I), dtype=torch.bfloat16, device=device)
        self.h = torch.empty((1, I), dtype=torch.bfloat16, device=device)

    def run(self, x, out):
        dv = self.dv
        if self.fused:
            self.mstack.forward(x, y=out)
            return
        cur = x
        for l, ((sg, pg), (su, pu), (sd, pd)) in enumerate(self.layers):
            dv.dvssq_linear_forward(sg, pg, cur, y=self.g, y_dtype=dv.Y_BF16, workspace=self.ws)
            dv.dvssq_linear_forward(su, pu, cur, y=self.u, y_dtype=dv.Y_BF16, workspace=self.ws)
            dv.dvssq_gelu_mul(self.g, self.u, self.h)
            dv.dvssq_linear_forward(sd, pd, self.h, y=out, y_dtype=dv.Y_BF16, workspace=self.ws)
            cur = out

    def step_slot(self, i):
        self.run(self.x0, self.x)

    def step(self):
        self.step_slot(0)

    def bytes_per_step(self):
        return sum(packed_bytes(sh.M, sh.K, sh.rank, sh.n_sal) for mats in self.layers
                   for sh, _ in mats)

    def launches_per_step(self):
        return 1 if self.fused else self.nl * (3 * 2 + 1)

    def kernel_work(self, name):
        if name == "mlp_stack":
            return self.bytes_per_step()
        # average algorithmic bytes per launch over the stack's launches
        shapes = [sh for mats in self.layers for sh, _ in mats]
        per = [kernel_bytes(name, sh.M, sh.K, sh.rank, sh.n_sal, 1) for sh in shapes]
        if name == "gelu_mul":
            return 3 * self.I * 2
        if any(v is None for v in per):
            return None
        return sum(per) / len(per)

    def config(self):
        return {"workload": self.name, "layers": self.nl, "hidden": self.H, "intermediate": self.I,
                "block": 256, "rank": "16 (layers 0-13, 29-35), 24 (14-28)",
                "n_sal": "K/8 per matrix", "tokens": 1,
                "step": (f"dvssq_mlp_stack_forward: the {self.nl} blocks in one cooperative launch"
                         if self.fused else
                         f"{self.nl} x (dvssq_linear_forward gate, up -> dvssq_gelu_mul -> down)")
                        + ", BF16 hidden states, one CUDA graph per token",
                "packed_bytes_per_token": self.bytes_per_step(),
                "l2": "1.9 GB of packed weights per token > 126 MB L2",
                "lowrank_factors": "seeded synthetic U, V (values do not change the work)",
                "parallelism": "replica per GPU"}

    # ---- end-to-end: token in from pinned host memory, hidden state back ----
    def e2e_setup(self, synth):
        torch = self.torch
        self.hx = synth.activations(1, self.H, seed=9, n_outlier=13,
                                    outlier_scale=25.0).pin_memory()
        self.hy = torch.empty((1, self.H), dtype=torch.bfloat16).pin_memory()
        self.dx = torch.empty((1, self.H), dtype=torch.bfloat16, device=self.device)

    def e2e_step(self):
        self.dx.copy_(self.hx, non_blocking=True)
        self.run(self.dx, self.x)
        self.hy.copy_(self.x, non_blocking=True)

    def e2e_bytes(self):
        return self.H * 2, self.H * 2

    # ---- the oracle on the host cores: forwards of one gate matrix ----
    def oracle_sample(self, O, synth):
        H, I = self.H, self.I
        W = synth.weight(I, H, seed=77, n_outlier_cols=2, outlier_scale=15.0)
        enc = O.encode(O.torch_bf16_to_f64(W), synth.act_scale(H, seed=77).numpy(), 256, 0,
                       with_svd=False)
        U, V = synth.lowrank_factors(I, H, 16, seed=78)
        Uf, Vf = O.torch_bf16_to_f64(U), O.torch_bf16_to_f64(V)
        x = O.torch_bf16_to_f64(synth.activations(1, H, seed=79))
        self._oracle_bytes = packed_bytes(I, H, 16, H // 8)
        self.oracle_what = "forward(s) of one 10240 x 2560 gate matrix (packed bytes per forward)"

        def step():
            O.forward(enc, x, U=Uf, V=Vf)
        return step


class StackChainStep(StackStep):
    """The same stack as 108 single-layer forwards and 36 gelu_mul launches."""
    name = "spark_mlp_stack_36x(gate,up,down)_T1_chain"
    fused = False


class ForwardLeg:
    """Forwards of one synthetic layer at fixed token counts, on rotating
    pre-encoded copies whose total size exceeds L2 (decode GEMV for T <= 16,
    the tensor-core GEMM above).  Unit: GB/s of packed bytes per forward for
    the decode path, TFLOP/s (2 T M K + 2 T r (K + M)) for the GEMM path."""

    def __init__(self, dv, synth, torch, rank_id, device, wl_name, tokens, n_copies):
        self.dv, self.torch = dv, torch
        wl = synth.WORKLOADS[wl_name]
        self.wl, self.tokens, self.n_copies = wl, tuple(tokens), n_copies
        M, K, r, n = wl.M, wl.K, wl.rank, wl.n_sal
        self.M, self.K, self.r, self.n = M, K, r, n
        self.shape = dv.Shape.make(M, K, wl.block, r, n)
        self.name = f"{wl_name}_{M}x{K}_r{r}_fwd_T" + "+".join(str(t) for t in tokens)
        self.unit = "TFLOP/s" if min(tokens) > 16 else "GB/s"
        ws = torch.empty(dv.dvssq_encode_workspace_size(self.shape), dtype=torch.uint8,
                         device=device)
        self.copies = []
        for c in range(n_copies):
            off = 1000 * rank_id + c
            U, V = synth.lowrank_factors(M, K, r, seed=wl.seed + 7 + off)
            packed = dv.PackedWeights.empty(self.shape, device, U=U.to(device), V=V.to(device))
            dv.dvssq_encode(self.shape, wl.weight(seed_offset=off).to(device),
                            wl.act_scale(seed_offset=off).to(device), packed, workspace=ws)
            self.copies.append(packed)
        self.x = {T: wl.activations(T, seed_offset=rank_id).to(device) for T in tokens}
        self.ws = {T: torch.empty(max(1, dv.dvssq_forward_workspace_size(self.shape, T)),
                                  dtype=torch.uint8, device=device) for T in tokens}
        self.y = {T: torch.empty((T, M), dtype=torch.float32, device=device) for T in tokens}
        self.i = 0

    @property
    def graph_slots(self):
        return self.n_copies

    def step_slot(self, i):
        packed = self.copies[i % self.n_copies]
        for T in self.tokens:
            self.dv.dvssq_linear_forward(self.shape, packed, self.x[T], y=self.y[T],
                                         workspace=self.ws[T])

    def step(self):
        self.step_slot(self.i)
        self.i += 1

    def bytes_per_step(self):
        return len(self.tokens) * packed_bytes(self.M, self.K, self.r, self.n)

    def work_per_step(self):
        M, K, r = self.M, self.K, self.r
        return sum(2.0 * T * M * K + 2.0 * T * r * (K + M) for T in self.tokens)

    def kernel_work(self, name):
        if name == "pre_gemm":
            return self.work_per_step()
        T = max(self.tokens)
        salp = (self.n + 63) // 64 * 64
        kc = self.K + salp + 64
        if name == "pre_act":
            return T * self.K * 2 + T * kc * 2
        if name == "pre_mat":
            return packed_bytes(self.M, self.K, self.r, self.n) + self.M * kc * 2
        return kernel_bytes(name, self.M, self.K, self.r, self.n, T)

    def config(self):
        mb = packed_bytes(self.M, self.K, self.r, self.n) / 1e6
        return {"workload": self.name, "M": self.M, "K": self.K, "block": self.wl.block,
                "rank": self.r, "n_sal": self.n, "tokens": list(self.tokens),
                "l2": f"{self.n_copies} rotating encoded layers (~{self.n_copies * mb:.0f} MB) "
                      "> 126 MB L2",
                "lowrank_factors": "seeded synthetic U, V (values do not change the work)"}


class MaterializeLeg:
    """dvssq_materialize of the Spark down_proj (2560 x 10240, r = 16): the
    dense BF16 W_eff in the original domain, on rotating packed copies.
    Unit: GB/s of packed bytes read + BF16 bytes written."""

    name = "spark_down_proj_2560x10240_r16_materialize"

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv = dv
        self.fw = ForwardLeg(dv, synth, torch, rank_id, device, "spark_down", (1,), 8)
        self.M, self.K, self.r, self.n = self.fw.M, self.fw.K, self.fw.r, self.fw.n
        self.W = torch.empty((self.M, self.K), dtype=torch.bfloat16, device=device)
        self.i = 0

    graph_slots = 8

    def step_slot(self, i):
        self.dv.dvssq_materialize(self.fw.shape, self.fw.copies[i % 8], out=self.W)

    def step(self):
        self.step_slot(self.i)
        self.i += 1

    def bytes_per_step(self):
        return packed_bytes(self.M, self.K, self.r, self.n) + self.M * self.K * 2

    def kernel_work(self, name):
        return self.bytes_per_step() if name == "materialize" else None

    def config(self):
        return {"workload": self.name, "M": self.M, "K": self.K, "block": 256, "rank": self.r,
                "n_sal": self.n, "l2": "8 rotating packed layers (141 MB) > 126 MB L2; the "
                "52 MB BF16 output is rewritten every step"}


class LowrankLeg:
    """dvssq_lowrank of the Spark down_proj residual (2560 x 10240 FP32, rank
    16, 4 power iterations): the truncated SVD of the encoder on the GPU.
    Unit: GB/s of residual bytes read by the products with R (each launch of
    lr_mul reads R once: 2 (iters + 1) + 1 = 11 reads per call)."""

    name = "spark_down_proj_2560x10240_lowrank_r16_q4"
    iters = 4

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv = dv
        wl = synth.WORKLOADS["spark_down"]
        self.M, self.K, self.r = wl.M, wl.K, 16
        shape = dv.Shape.make(wl.M, wl.K, wl.block, 0)
        packed = dv.PackedWeights.empty(shape, device)
        self.R = torch.empty((wl.M, wl.K), dtype=torch.float32, device=device)
        dv.dvssq_encode(shape, wl.weight(seed_offset=rank_id).to(device),
                        wl.act_scale(seed_offset=rank_id).to(device), packed, resid=self.R)
        self.U = torch.empty((wl.M, 16), dtype=torch.bfloat16, device=device)
        self.V = torch.empty((16, wl.K), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(dv.dvssq_lowrank_workspace_size(wl.M, wl.K, 16), dtype=torch.uint8,
                              device=device)

    graph_slots = 1

    def step_slot(self, i):
        self.dv.dvssq_lowrank(self.R, 16, iters=self.iters, seed=5, U=self.U, V=self.V,
                              workspace=self.ws)

    def step(self):
        self.step_slot(0)

    def bytes_per_step(self):
        return (2 * (self.iters + 1) + 1) * self.M * self.K * 4

    def kernel_work(self, name):
        return self.M * self.K * 4 if name == "lr_mul" else None

    def config(self):
        return {"workload": self.name, "M": self.M, "K": self.K, "rank": 16,
                "iters": self.iters, "oversampling": 16,
                "l2": "the 105 MB FP32 residual is read 11 times per call; partly from L2"}


class BssAttentionLeg:
    """KV-BSS decode attention of the Spark attention shape: 16 query heads, 4
    KV heads, head_dim 256, one query token per sequence over a 32768-token
    BF16 KV cache, batch 4 (K + V = 537 MB > L2).  Seeded N(0, 1) tensors,
    so the truncation drops few keys and every V row is read.
    Unit: GB/s of K and V bytes."""

    name = "spark_attention_kv_bss_B4_Hq16_Hkv4_d256_L32768"

    def __init__(self, dv, synth, torch, rank_id, device):
        self.dv = dv
        self.B, self.Hq, self.Hkv, self.d, self.L = 4, 16, 4, 256, 32768
        gen = torch.Generator(device=device)
        gen.manual_seed(1234 + rank_id)
        mk = lambda *s: torch.randn(s, generator=gen, device=device).to(torch.bfloat16)
        self.q = mk(self.B, self.Hq, self.d)
        self.k = mk(self.B, self.Hkv, self.L, self.d)
        self.v = mk(self.B, self.Hkv, self.L, self.d)
        self.out = torch.empty((self.B, self.Hq, self.d), dtype=torch.float32, device=device)
        shape = dv.AttnShape(self.B, self.Hq, self.Hkv, self.d, self.L, 1.10, 12.0)
        self.ws = torch.empty(dv.dvssq_bss_attention_workspace_size(shape), dtype=torch.uint8,
                              device=device)

    graph_slots = 1

    def step_slot(self, i):
        self.dv.dvssq_bss_attention(self.q, self.k, self.v, out=self.out, workspace=self.ws)

    def step(self):
        self.step_slot(0)

    def kv_bytes(self):
        return self.B * self.Hkv * self.L * self.d * 2

    def bytes_per_step(self):
        return 2 * self.kv_bytes()

    def kernel_work(self, name):
        logits = self.B * self.Hq * self.L * 4
        if name == "bss_logits":
            return self.kv_bytes() + logits
        if name == "bss_pv":
            return self.kv_bytes() + logits
        return None

    def config(self):
        return {"workload": self.name, "batch": self.B, "q_heads": self.Hq,
                "kv_heads": self.Hkv, "head_dim": self.d, "ctx": self.L, "tau": 1.10,
                "haze": 12.0, "l2": "537 MB of K and V per step > 126 MB L2"}


# Legs of the metric timed in the default single-GPU run besides the headline:
# (name, constructor).  Each is built, timed and freed in turn.
def leg_specs():
    def fwd(wl, tokens, copies):
        return lambda dv, synth, torch, r, d: ForwardLeg(dv, synth, torch, r, d, wl, tokens, copies)
    return [
        ("decode_T1", fwd("spark_down", (1,), 8)),
        ("decode_T16", fwd("spark_down", (16,), 8)),
        ("stack", StackStep),
        ("prefill", PrefillStep),
        ("bulk_encode", BulkEncodeStep),
        ("materialize", MaterializeLeg),
        ("lowrank", LowrankLeg),
        ("bss_attention", BssAttentionLeg),
        ("minicpm_k_T1", fwd("minicpm_k", (1,), 192)),
        ("minicpm_k_T8", fwd("minicpm_k", (8,), 192)),
        ("minicpm_k_T64", fwd("minicpm_k", (64,), 192)),
        ("minicpm_up_T1", fwd("minicpm_up", (1,), 16)),
        ("minicpm_up_T8", fwd("minicpm_up", (8,), 16)),
        ("minicpm_up_T64", fwd("minicpm_up", (64,), 16)),
    ]


WORKLOADS = {"spark_down": SparkDownStep, "decode": DecodeStep, "prefill": PrefillStep,
             "bulk_encode": BulkEncodeStep, "stack": StackStep, "stack_chain": StackChainStep}


# -------------------------------------------------------------------- main --

def threads_used():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_oracle(work, O, synth, budget_s=20.0, min_steps=1, max_steps=10):
    step = work.oracle_sample(O, synth)
    t0 = time.perf_counter()
    n = 0
    while n < min_steps or (time.perf_counter() - t0 < budget_s and n < max_steps):
        step()
        n += 1
    dt = time.perf_counter() - t0
    return n, dt


def max_over_ranks(x, world, device):
    """The largest value of x over the ranks (the job's time is its slowest
    rank's).  Every rank must call it, in the same order."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank_step, ms_step, scale):
    """Whole-job throughput: every rank processes units_per_rank_step per
    step (weak scaling), and a step takes ms_step on the slowest rank."""
    return world * units_per_rank_step / (ms_step * 1e-3) / scale


def cpu_info():
    """(logical CPUs of the host, CPU model name)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def measure(work, dv, torch, steps, warmup, world, device, local, key, use_graphs=True):
    """Time one workload: W warm-up steps, K timed steps (CUDA graph replay
    when the workload has graph slots) bracketed by a barrier and a device
    synchronize, clocks sampled meanwhile; then the same K steps eagerly with
    per-launch CUDA events for the per-kernel times and the roofline of the
    dominant kernel."""
    unit = getattr(work, "unit", "GB/s")
    W = max(3, warmup)
    for _ in range(W):
        work.step()
    torch.cuda.synchronize()
    dv.dvssq_device_error(clear=True)

    # one CUDA graph per rotation slot: the timed region replays the same
    # launches without the host in the loop
    graphs = []
    n_slots = getattr(work, "graph_slots", 0)
    if n_slots and use_graphs:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for slot in range(n_slots):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=side):
                    work.step_slot(slot)
                graphs.append(g)
        torch.cuda.current_stream().wait_stream(side)
        for i in range(W):
            graphs[i % n_slots].replay()
        torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(steps):
            if graphs:
                graphs[i % n_slots].replay()
            else:
                work.step()
        stop.record(stream)
        barrier()
    ms = max_over_ranks(start.elapsed_time(stop), world, device)
    err = dv.dvssq_device_error(clear=True)
    del graphs
    ms_step = ms / steps
    if unit == "TFLOP/s":
        bytes_step = None
        value = job_throughput(world, work.work_per_step(), ms_step, 1e12)
    else:
        bytes_step = work.bytes_per_step()
        value = job_throughput(world, bytes_step, ms_step, 1e9)

    # per-kernel device times: the same K steps again with events around each launch
    dv.dvssq_profile_reset()
    dv.dvssq_profile_enable(True)
    for _ in range(steps):
        work.step()
    torch.cuda.synchronize()
    dv.dvssq_profile_collect()
    dv.dvssq_profile_enable(False)
    prof = dv.dvssq_profile_read()
    launches_measured = sum(c for c, _ in prof.values())
    pk, pk_kind = peaks()
    # a kernel timed within a run of milliseconds runs at the burst tensor rate
    tpk = pk["bf16_tflops"]
    kernels = {}
    tot_ms = sum(v[1] for v in prof.values())
    kb_fn = getattr(work, "kernel_work", None) or (
        lambda name: kernel_bytes(name, work.M, work.K, work.r, work.n, 16))
    for name, (cnt, kms) in prof.items():
        avg = kms / cnt
        ent = {"launches": cnt, "avg_us": round(avg * 1e3, 3), "share": round(kms / tot_ms, 4)}
        b = kb_fn(name)
        if b is not None:
            if name == "pre_gemm":
                tfs = b / (avg * 1e-3) / 1e12
                ent.update(flops=b, tflops=round(tfs, 1), frac=round(tfs / tpk, 4))
            else:
                gbs = b / (avg * 1e-3) / 1e9
                ent.update(bytes=b, gbs=round(gbs, 1), frac=round(gbs / pk["hbm_gbs"], 4))
        kernels[name] = ent
    # dominant kernel among those with an algorithmic work count
    dom = max((kv for kv in prof.items() if kb_fn(kv[0]) is not None), key=lambda kv: kv[1][1])[0]
    db = kb_fn(dom)
    dom_avg_ms = prof[dom][1] / prof[dom][0]
    if dom == "pre_gemm":
        achieved = db / (dom_avg_ms * 1e-3) / 1e12
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": tpk,
                    "peak_source": pk_kind + " bf16 burst (a kernel timed within a short run; "
                                             "f16 has the same dense rate)",
                    "unit": "TFLOP/s", "frac": round(achieved / tpk, 4),
                    "traffic": dram_traffic(dom, key),
                    "algorithmic_flops_per_launch": db}
    else:
        achieved = db / (dom_avg_ms * 1e-3) / 1e9
        roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": pk["hbm_gbs"], "peak_source": pk_kind, "unit": "GB/s",
                    "frac": round(achieved / pk["hbm_gbs"], 4),
                    "traffic": dram_traffic(dom, key),
                    "algorithmic_bytes_per_launch": db}
    # the task's bars: decode GEMV >= 0.70 of HBM, prefill GEMM >= 0.50 of the BF16 peak
    target = ROOFLINE_TARGETS.get(dom)
    if target is not None:
        roofline["target_frac"] = target
        roofline["frac_of_target"] = round(roofline["frac"] / target, 4)
    return dict(ms_step=ms_step, value=value, unit=unit, bytes_step=bytes_step, kernels=kernels,
                roofline=roofline, launches=launches_measured, err=err, clocks=clk.summary(),
                W=W, barrier=barrier, stream=stream)


def run_legs(dv, synth, torch, rank, device, local, steps, warmup, only=()):
    """Every leg of the metric besides the headline, each timed on its own."""
    legs = {}
    for name, ctor in leg_specs():
        if only and name not in only:
            continue
        work = ctor(dv, synth, torch, rank, device)
        n = steps if name not in ("bulk_encode", "stack") else max(5, steps // 3)
        r = measure(work, dv, torch, n, warmup, 1, device, local, name)
        ent = {"workload": work.config()["workload"], "value": round(r["value"], 2),
               "unit": r["unit"], "ms_per_step": round(r["ms_step"], 5), "steps": n,
               "warmup": r["W"], "roofline": r["roofline"], "kernels": r["kernels"],
               "gpu_launches": r["launches"], "device_error_word": r["err"],
               "clocks": r["clocks"], "l2": work.config().get("l2")}
        if r["unit"] == "GB/s":
            ent["frac_of_hbm"] = round(r["value"] / peaks()[0]["hbm_gbs"], 4)
        legs[name] = ent
        del work
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return legs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="spark_down")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graphs", action="store_true")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the other legs of the metric (timed by default on one GPU)")
    ap.add_argument("--legs", default="",
                    help="comma-separated subset of the legs to time (default: all)")
    ap.add_argument("--layers", type=int, default=36,
                    help="blocks of the stack workloads (36 is the full model; fewer for profiling)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    import torch.distributed as dist
    import mixed_precision_weight_b200 as pkg
    from mixed_precision_weight_b200 import synth
    dv = pkg.binding

    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(device))
    StackStep.n_layers = args.layers
    work = WORKLOADS[args.workload](dv, synth, torch, rank, device)
    r = measure(work, dv, torch, args.steps, args.warmup, world, device, local, args.workload,
                use_graphs=not args.no_graphs)
    unit, value, ms_step, bytes_step = r["unit"], r["value"], r["ms_step"], r["bytes_step"]
    kernels = r["kernels"]
    cfg = work.config()
    barrier, stream = r["barrier"], r["stream"]
    # the decode GEMV's own roofline (the headline HBM-bound kernel)
    dm = kernels.get("dec_row") or kernels.get("dec_main") or kernels.get("mlp_stack")

    # end-to-end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e and hasattr(work, "e2e_step"):
        work.e2e_setup(synth)
        for _ in range(2):
            work.e2e_step()
        torch.cuda.synchronize()
        e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        barrier()
        e_start.record(stream)
        for _ in range(n_e2e):
            work.e2e_step()
        e_stop.record(stream)
        barrier()
        ems = max_over_ranks(e_start.elapsed_time(e_stop) / n_e2e, world, device)
        h2d, d2h = work.e2e_bytes()
        e2e = {"value": round(job_throughput(world, bytes_step, ems, 1e9), 2), "unit": "GB/s",
               "ms_per_step": round(ems, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and hasattr(work, "oracle_sample"):
        from oracle import dvssq_oracle as O
        nst, dt = run_oracle(work, O, synth)
        sample_bytes = getattr(work, "_oracle_bytes", None) or bytes_step
        what = getattr(work, "oracle_what", "full step(s) of the same workload "
                                            "(encode without SVD + 2 forwards)")
        nproc, model = cpu_info()
        cpu = {"value": round(sample_bytes * nst / dt / 1e9, 4), "unit": "GB/s",
               "cores": threads_used(), "nproc": nproc, "cpu_model": model, "kind": "oracle",
               "sample": f"{nst} {what} on the host, {dt:.1f} s; numpy fp64 with "
                         f"{threads_used()} BLAS threads for the matrix products, "
                         "single-threaded Python loops for the sums of squares"}

    legs = None
    if world == 1 and args.workload == "spark_down" and not args.no_legs:
        del work
        torch.cuda.empty_cache()
        only = tuple(x for x in args.legs.split(",") if x)
        legs = run_legs(dv, synth, torch, rank, device, local, args.steps, args.warmup, only)

    line = {"metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": r["W"], "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64+fp16",
            "data": "synthetic (seeded N(0,0.02) weights with outlier columns, N(0,1) tokens)",
            "config": cfg,
            "roofline": r["roofline"], "kernels": kernels,
            "decode_gemv": dm, "gpu_launches": r["launches"],
            "e2e": e2e, "cpu_baseline": cpu, "device_error_word": r["err"],
            "clocks": r["clocks"], "legs": legs}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def run_reference(args, world, rank):
    """The oracle timed as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    import torch  # noqa: F401  (synth uses torch for BF16 rounding)
    from mixed_precision_weight_b200 import synth
    from oracle import dvssq_oracle as O

    base = WORKLOADS.get(args.workload)
    if base not in (SparkDownStep, DecodeStep):
        print(json.dumps({"impl": "reference", "unavailable":
                          f"the oracle arm times the spark_down and decode workloads; "
                          f"{args.workload} has no host step of its own"}))
        return

    class _W(base):
        def __init__(self):
            wl = synth.WORKLOADS["spark_down"]
            self.wl = wl
            self.M, self.K, self.r, self.n = wl.M, wl.K, wl.rank, wl.n_sal
    work = _W()
    step = work.oracle_sample(O, synth)
    for _ in range(max(0, min(args.warmup, 1))):
        step()
    t0 = time.perf_counter()
    nst = max(1, min(args.steps, 3))
    for _ in range(nst):
        step()
    dt = time.perf_counter() - t0
    v = work.bytes_per_step() * nst / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
            "n_gpus": world, "steps": nst, "warmup": min(args.warmup, 1),
            "ms_per_step": round(dt / nst * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": work.config(),
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "kind": "oracle",
                             "cores": threads_used(),
                             "sample": f"{nst} full steps of the workload on the host"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
