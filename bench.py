#!/usr/bin/env python
"""Throughput of the tensor-parallel layers on B200 (one JSON line on rank 0).

One step = one pass of the whole hot path over one batch of seeded synthetic
input, all through the library's C ABI on the current stream:
  1. TP-MLP forward + backward, M=4096 (b=2, s=2048), h=4096, ffn=16384, N=8
     (column GEMM + bias + GeLU, row GEMM with the fused shard sum, dGeLU GEMM,
     dB, dA + dbias, dX with the fused shard sum): 3.2985 TFLOP;
  2. attention projections of the GPT-2 1.5B layer slice (M=4096, h=1600,
     25 heads over N=4 shards as 7/6/6/6): column-parallel QKV and
     row-parallel output projection, forward + backward: 0.2516 TFLOP;
  3. vocabulary path, T=16384 (b=8, s=2048), v=50304 over N=8, h=4096:
     embedding lookup, logits = H·Eᵀ (fp32, 6.752 TFLOP), softmax
     cross-entropy with loss, loss_sum, in-place dlogits and arg-max;
  4. vocabulary backward: the cross-entropy gradient in bf16, dH = dlogits·E
     and dE = dlogitsᵀ·H (13.5 TFLOP), and the input-embedding scatter-add
     onto that dE (the gradient of the shared table).

value = TP-MLP forward+backward TFLOP/s (all ranks' FLOPs / max-over-ranks
device time of the MLP part); the cross-entropy half of the metric is the
"vocab_xent" object (tokens/s and HBM GB/s).  Times are CUDA events on the
launching stream; every input set is far larger than the 126 MB L2.

--impl reference times the fp64 CPU oracle (the reference arm of this
build) on a bounded row sample of the same TP-MLP workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TP-MLP fwd+bwd bf16 TFLOP/s & % tensor peak; vocab-xent tokens/s & % HBM"

# workloads (sizes only)
MLP = dict(M=4096, h=4096, F=16384, N=8, w_std=0.006)
PROJ = dict(M=4096, h=1600, n_heads=25, head_dim=64, N=4)
VOC = dict(T=16384, v=50304, h=4096, N=8, e_std=0.02)

MLP_FLOP = 12.0 * MLP["M"] * MLP["h"] * MLP["F"]                       # 6 GEMMs x 2MhF
PROJ_FLOP = 6.0 * PROJ["M"] * PROJ["h"] * 3 * PROJ["h"] + 6.0 * PROJ["M"] * PROJ["h"] ** 2
LOGITS_FLOP = 2.0 * VOC["T"] * VOC["v"] * VOC["h"]
ATTN_FLOP = 4.0 * 4 * 25 * 64 * (1024 * 1025 / 2)                      # b=4, 25 heads, s=1024
LN_FWD_BYTES = 8.0 * 4096 * 1600
LN_BWD_BYTES = 10.0 * 4096 * 1600
LOGITS_BWD_FLOP = 2.0 * LOGITS_FLOP
# algorithmic bytes: read + write every logit once, plus targets / loss / argmax
XENT_BYTES = 2 * 4 * VOC["T"] * VOC["v"] + VOC["T"] * (8 + 4 + 4)
EMBED_BYTES = 2 * 2 * VOC["T"] * VOC["h"] + 8 * VOC["T"]
# bf16-gradient cross-entropy: read fp32 logits, write bf16 dlogits
XENT_BF16_BYTES = (4 + 2) * VOC["T"] * VOC["v"] + VOC["T"] * (8 + 4 + 4)

SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


KERNEL_SOURCES = ("linear_layers_b200/csrc/gemm_tc.cu", "linear_layers_b200/csrc/sm100_ptx.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_tc_traffic.json")


def kernel_source_hash():
    import hashlib

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _roofline_traffic():
    """DRAM bytes per GEMM launch from the committed ncu capture, or None when
    the capture is missing or the kernel sources changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        if t.get("source_sha256") != kernel_source_hash():
            return None, "kernel changed since the ncu capture"
        return float(t["dram_bytes_per_launch"]), t.get("command", "")
    except Exception:
        return None, "no ncu capture"


def _dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.skip = 0
        self.path = os.path.join("/tmp", f"tp_clocks_{os.getpid()}.csv")

    def _lines(self) -> int:
        try:
            with open(self.path) as f:
                return sum(1 for line in f if line.endswith("\n"))
        except OSError:
            return 0

    def __enter__(self):
        """Starts sampling and returns once the first sample is written (at
        most 5 s), so that a short timed region that follows is covered."""
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            t0 = time.perf_counter()
            while self._lines() == 0 and time.perf_counter() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def mark(self):
        """Samples written before this call (start-up, warm-up) are left out."""
        self.skip = self._lines()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for i, line in enumerate(f):
                if i < self.skip:
                    continue
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        # median over samples under load (clock above idle)
        loaded = [x for x in sm if x > 500] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def _prepare(dev, parts):
    import torch

    import linear_layers_b200 as tpl
    import tp_inputs

    g = pr = vo = None
    bf = dict(dtype=torch.bfloat16, device=dev)
    if any(p.startswith("mlp") or p.endswith("_gemm") for p in parts):
        g = _prepare_mlp(dev, tpl, tp_inputs, torch, bf)
    if any(p in parts for p in ("proj", "attn_fwd", "attn_bwd", "ln_fwd", "ln_bwd")):
        pr = _prepare_proj(dev, tpl, tp_inputs, torch, bf)
    if any(p in parts for p in ("embed", "logits", "xent", "xent_bf16", "logits_bwd", "embed_bwd",
                                "lxent_fwd", "lxent_dlogits")):
        vo = _prepare_vocab(dev, tpl, tp_inputs, torch, bf, "logits" not in parts)
    return g, pr, vo


def _prepare_mlp(dev, tpl, tp_inputs, torch, bf):
    m = tp_inputs.mlp_inputs(MLP["M"], MLP["h"], MLP["F"], w_std=MLP["w_std"], seed=0)
    g = {k: v.to(dev) for k, v in m.items()}
    M, h, F = MLP["M"], MLP["h"], MLP["F"]
    g.update(U=torch.empty(M, F, **bf), Y=torch.empty(M, F, **bf), Z=torch.empty(M, h, **bf),
             dU=torch.empty(M, F, **bf), dX=torch.empty(M, h, **bf), dA=torch.empty(h, F, **bf),
             dB=torch.empty(F, h, **bf), dbias=torch.empty(F, dtype=torch.float32, device=dev))
    g["ws_f"] = torch.empty(max(1, tpl.tp_workspace_bytes(tpl.OP_MLP_FWD, M, h, F, MLP["N"])),
                            dtype=torch.uint8, device=dev)
    g["ws_b"] = torch.empty(max(1, tpl.tp_workspace_bytes(tpl.OP_MLP_BWD, M, h, F, MLP["N"])),
                            dtype=torch.uint8, device=dev)
    return g


def _prepare_proj(dev, tpl, tp_inputs, torch, bf):
    p = tp_inputs.attn_proj_inputs(PROJ["M"], PROJ["h"], PROJ["n_heads"], PROJ["head_dim"],
                                   PROJ["N"], seed=0)
    pr = {k: v.to(dev) for k, v in p.items()}
    heads = tp_inputs.head_split(PROJ["n_heads"], PROJ["N"])
    qkv_offs, ctx_offs = [0], [0]
    for nh in heads:
        qkv_offs.append(qkv_offs[-1] + 3 * nh * PROJ["head_dim"])
        ctx_offs.append(ctx_offs[-1] + nh * PROJ["head_dim"])
    pr["qkv_offs"], pr["ctx_offs"] = qkv_offs, ctx_offs
    Mp, hp = PROJ["M"], PROJ["h"]
    pr.update(QKV=torch.empty(Mp, 3 * hp, **bf), dXq=torch.empty(Mp, hp, **bf),
              dWq=torch.empty(hp, 3 * hp, **bf), dbq=torch.empty(3 * hp, dtype=torch.float32, device=dev),
              Zo=torch.zeros(Mp, hp, **bf), dctx=torch.zeros(Mp, hp, **bf), dWo=torch.empty(hp, hp, **bf),
              ctx_attn=torch.empty(Mp, hp, **bf),
              attn_lse=torch.empty(Mp // 1024, PROJ["n_heads"], 1024, dtype=torch.float32, device=dev),
              dqkv_attn=torch.empty(Mp, 3 * hp, **bf),
              attn_ws=torch.empty(tpl.tp_workspace_bytes(tpl.OP_ATTENTION_BWD, Mp, PROJ["n_heads"], 64,
                                                         PROJ["N"]), dtype=torch.uint8, device=dev))
    # the residual step after the output projection: hs = X + dropout(Zo + b), y = LN(hs)
    gl = torch.Generator().manual_seed(5)
    pr.update(ln_bias=(0.1 * torch.randn(hp, generator=gl)).to(**bf),
              ln_gamma=(1 + 0.1 * torch.randn(hp, generator=gl)).to(**bf),
              ln_beta=(0.1 * torch.randn(hp, generator=gl)).to(**bf),
              ln_hs=torch.empty(Mp, hp, **bf), ln_y=torch.empty(Mp, hp, **bf),
              ln_mean=torch.empty(Mp, dtype=torch.float32, device=dev),
              ln_rstd=torch.empty(Mp, dtype=torch.float32, device=dev),
              ln_dx=torch.empty(Mp, hp, **bf), ln_dres=torch.empty(Mp, hp, **bf),
              ln_dg=torch.empty(hp, dtype=torch.float32, device=dev),
              ln_db=torch.empty(hp, dtype=torch.float32, device=dev),
              ln_dbias=torch.empty(hp, dtype=torch.float32, device=dev),
              ln_ws=torch.empty(tpl.tp_workspace_bytes(tpl.OP_SP_LN_BWD, Mp, hp, hp, PROJ["N"]),
                                dtype=torch.uint8, device=dev))
    # the attention core reads the QKV projection of these inputs
    tpl.tp_col_linear_fwd(pr["X"], pr["Wqkv"], pr["bqkv"], PROJ["N"], shard_offsets=pr["qkv_offs"],
                          Y=pr["QKV"])
    torch.cuda.synchronize(dev)
    pr["ws_q"] = torch.empty(max(1, tpl.tp_workspace_bytes(tpl.OP_COL_LINEAR_BWD, Mp, hp, 3 * hp,
                                                           PROJ["N"])), dtype=torch.uint8, device=dev)
    pr["ws_o"] = torch.empty(max(1, tpl.tp_workspace_bytes(tpl.OP_ROW_LINEAR_FWD, Mp, hp, hp,
                                                           PROJ["N"])), dtype=torch.uint8, device=dev)
    return pr


def _prepare_vocab(dev, tpl, tp_inputs, torch, bf, fill_logits):
    vi = tp_inputs.vocab_inputs(VOC["T"], VOC["v"], VOC["h"], e_std=VOC["e_std"], seed=0)
    vo = {k: x.to(dev) for k, x in vi.items()}
    T, v = VOC["T"], VOC["v"]
    vb = tp_inputs.vocab_bwd_inputs(T, v, VOC["h"], seed=1)
    vo.update(dout=vb["dout"].to(dev), dlogits_bf=torch.empty(T, v, **bf),
              dH=torch.empty(T, VOC["h"], **bf),
              dE=torch.empty(v, VOC["h"], dtype=torch.float32, device=dev),
              ws_eb=torch.empty(max(1, tpl.tp_workspace_bytes(tpl.OP_EMBED_BWD, T, VOC["h"], v,
                                                              VOC["N"])),
                                dtype=torch.uint8, device=dev))
    vo.update(lse=torch.empty(T, dtype=torch.float32, device=dev),
              ws_lx=torch.empty(tpl.tp_workspace_bytes(tpl.OP_LINEAR_XENT, T, VOC["h"], v, VOC["N"]),
                                dtype=torch.uint8, device=dev))
    vo.update(emb=torch.empty(T, VOC["h"], **bf), logits=torch.empty(T, v, dtype=torch.float32, device=dev),
              loss=torch.empty(T, dtype=torch.float32, device=dev),
              loss_sum=torch.empty(1, dtype=torch.float32, device=dev),
              argmax=torch.empty(T, dtype=torch.int32, device=dev))
    if fill_logits:   # the loss alone is timed: give it real logits once
        tpl.tp_logits_fwd(vo["H"], vo["E"], VOC["N"], logits=vo["logits"])
        torch.cuda.synchronize(dev)
    return vo


def _mlp_fwd(tpl, g, st):
    tpl.tp_mlp_fwd(g["X"], g["A"], g["bias"], g["B"], MLP["N"], U=g["U"], Y=g["Y"], Z=g["Z"],
                   ws=g["ws_f"], dev_status=st)


def _mlp_bwd(tpl, g, st):
    tpl.tp_mlp_bwd(g["X"], g["A"], g["B"], g["U"], g["Y"], g["dZ"], MLP["N"], dU=g["dU"],
                   dX=g["dX"], dA=g["dA"], dbias=g["dbias"], dB=g["dB"], ws=g["ws_b"], dev_status=st)


def _proj(tpl, pr, st):
    N = PROJ["N"]
    tpl.tp_col_linear_fwd(pr["X"], pr["Wqkv"], pr["bqkv"], N, shard_offsets=pr["qkv_offs"],
                          Y=pr["QKV"], dev_status=st)
    tpl.tp_col_linear_bwd(pr["X"], pr["Wqkv"], None, pr["dQKV"], N, shard_offsets=pr["qkv_offs"],
                          dX=pr["dXq"], dW=pr["dWq"], dbias=pr["dbq"], ws=pr["ws_q"], dev_status=st)
    tpl.tp_row_linear_fwd(pr["ctx"], pr["Wo"], N, shard_offsets=pr["ctx_offs"], Z=pr["Zo"],
                          ws=pr["ws_o"], dev_status=st)
    tpl.tp_row_linear_bwd(pr["ctx"], pr["Wo"], pr["dZ"], N, shard_offsets=pr["ctx_offs"],
                          dXin=pr["dctx"], dW=pr["dWo"], dev_status=st)


def _embed(tpl, vo, st):
    tpl.vp_embed(vo["ids"], vo["E"], VOC["N"], out=vo["emb"], dev_status=st)


def _logits(tpl, vo, st):
    tpl.tp_logits_fwd(vo["H"], vo["E"], VOC["N"], logits=vo["logits"], dev_status=st)


def _xent(tpl, vo, st):
    tpl.vp_xent(vo["logits"], vo["targets"], VOC["N"], grad_scale=1.0 / VOC["T"], loss=vo["loss"],
                loss_sum=vo["loss_sum"], dlogits=vo["logits"], argmax=vo["argmax"], dev_status=st)


def _xent_bf16(tpl, vo, st):
    tpl.vp_xent_bf16_grad(vo["logits"], vo["targets"], VOC["N"], grad_scale=1.0 / VOC["T"],
                          loss=vo["loss"], loss_sum=vo["loss_sum"], dlogits=vo["dlogits_bf"],
                          argmax=vo["argmax"], dev_status=st)


def _logits_bwd(tpl, vo, st):
    tpl.tp_logits_bwd(vo["dlogits_bf"], vo["H"], vo["E"], VOC["N"], dH=vo["dH"], dE=vo["dE"],
                      dev_status=st)


def _embed_bwd(tpl, vo, st):
    tpl.vp_embed_bwd(vo["ids"], vo["dout"], vo["dE"], VOC["N"], ws=vo["ws_eb"], dev_status=st)


def _mlp_bwd_rc(tpl, g, st):
    tpl.tp_mlp_bwd_recompute(g["X"], g["A"], g["B"], g["U"], g["dZ"], MLP["N"], Y=g["Y"],
                             dU=g["dU"], dX=g["dX"], dA=g["dA"], dbias=g["dbias"], dB=g["dB"],
                             ws=g["ws_b"], dev_status=st)


def _attn_fwd(tpl, pr, st):
    tpl.tp_attention_fwd(pr["QKV"], PROJ["M"] // 1024, 1024, PROJ["n_heads"], PROJ["N"],
                         causal=True, ctx=pr["ctx_attn"], lse=pr["attn_lse"], dev_status=st)


def _attn_bwd(tpl, pr, st):
    tpl.tp_attention_bwd(pr["QKV"], pr["ctx_attn"], pr["dZ"], pr["attn_lse"], PROJ["M"] // 1024,
                         1024, PROJ["n_heads"], PROJ["N"], causal=True, dQKV=pr["dqkv_attn"],
                         ws=pr["attn_ws"], dev_status=st)


LN_P, LN_SEED = 0.1, 1234


def _ln_fwd(tpl, pr, st):
    tpl.tp_sp_dropout_add_ln_fwd(pr["Zo"], pr["ln_bias"], pr["X"], pr["ln_gamma"], pr["ln_beta"],
                                 PROJ["N"], p=LN_P, seed=LN_SEED, offset=0, hs=pr["ln_hs"],
                                 y=pr["ln_y"], mean=pr["ln_mean"], rstd=pr["ln_rstd"], dev_status=st)


def _ln_bwd(tpl, pr, st):
    tpl.tp_sp_dropout_add_ln_bwd(pr["dZ"], pr["dctx"], pr["ln_hs"], pr["ln_gamma"], pr["ln_mean"],
                                 pr["ln_rstd"], PROJ["N"], p=LN_P, seed=LN_SEED, offset=0,
                                 dx=pr["ln_dx"], dresidual=pr["ln_dres"], dgamma=pr["ln_dg"],
                                 dbeta=pr["ln_db"], dbias=pr["ln_dbias"], ws=pr["ln_ws"],
                                 dev_status=st)


def _lxent_fwd(tpl, vo, st):
    tpl.tp_linear_xent_fwd(vo["H"], vo["E"], vo["targets"], VOC["N"], loss=vo["loss"],
                           loss_sum=vo["loss_sum"], lse=vo["lse"], argmax=vo["argmax"],
                           ws=vo["ws_lx"], dev_status=st)


def _lxent_dlogits(tpl, vo, st):
    tpl.tp_linear_xent_dlogits(vo["H"], vo["E"], vo["targets"], vo["lse"], VOC["N"],
                               grad_scale=1.0 / VOC["T"], dlogits=vo["dlogits_bf"], dev_status=st)


def _col_gemm(tpl, g, st):
    """The column GEMM of the h=4096 layer alone (U = X·A, no bias, no
    activation): the engine's main loop on the a2 shape, for profiling."""
    tpl.tp_col_linear_fwd(g["X"], g["A"], None, 1, Y=g["U"], dev_status=st)


def _cublas_gemm(torch, g):
    """torch.matmul (cuBLAS) on the same operands, for the same-box A/B."""
    torch.matmul(g["X"], g["A"], out=g["U"])


# the step: every row of the hot path
PARTS = ("mlp_fwd", "mlp_bwd", "proj", "embed", "logits", "xent")
# the vocabulary backward (the next row beyond the hot path), timed in its own
# loop after the step: logits (re-made, not reported) -> bf16-gradient loss ->
# dH, dE -> input-embedding scatter-add onto dE
BWD_PARTS = ("logits", "xent_bf16", "logits_bwd", "embed_bwd")
# output layer + loss without the logits matrix (the next row after that),
# also in its own loop: statistics GEMM + combine, then the recomputing
# gradient GEMM
FUSED_PARTS = ("lxent_fwd", "lxent_dlogits")
# the MLP backward with activation recompute (Y rebuilt from U), own loop
RECOMPUTE_PARTS = ("mlp_bwd_rc",)
# the attention core between the projections (b=4, s=1024, causal), own loop
ATTN_PARTS = ("attn_fwd", "attn_bwd")
# sequence-parallel dropout-add-LayerNorm after the output projection, own loop
LN_PARTS = ("ln_fwd", "ln_bwd")
# single GEMMs for profiling and the library A/B (partial runs only)
GEMM_PARTS = ("col_gemm", "cublas_gemm")


E2E_DATA = (("X", "dZ"), ("Z", "dX"))
E2E_ALL = (("X", "A", "bias", "B", "dZ"), ("Z", "dX", "dA", "dB", "dbias"))


def _e2e_mlp(tpl, torch, g, dev, steps, keys=E2E_DATA):
    """TP-MLP forward+backward through the public API from pinned host buffers.

    Every step copies its inputs keys[0] host->device and its results keys[1]
    device->host inside the timed region; tensors not named stay resident on
    the device (with E2E_DATA: the weights A, B, bias as model parameters, and
    the weight gradients dA, dB, dbias for an optimizer on the device).  The
    copies of neighbouring steps run on their own streams and overlap the
    compute of the current step (double-buffered device inputs and outputs).
    """
    in_keys, out_keys = keys
    host_in = {k: g[k].cpu().pin_memory() for k in in_keys}
    host_out = [{k: torch.empty(g[k].shape, dtype=g[k].dtype, pin_memory=True) for k in out_keys}
                for _ in range(2)]
    dev_in = [{k: torch.empty_like(g[k]) for k in in_keys} for _ in range(2)]
    dev_out = [{k: torch.empty_like(g[k]) for k in out_keys} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    st = tpl.new_status(dev)
    s_c = torch.cuda.current_stream(dev)
    s_h = torch.cuda.Stream(dev)
    s_d = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)

    def run(nsteps, timed):
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        h2d_done = [ev() for _ in range(nsteps)]
        comp_done = [ev() for _ in range(nsteps)]
        d2h_done = [ev() for _ in range(nsteps)]
        if timed:
            t0.record(s_h)
        for i in range(nsteps):
            b = i & 1
            with torch.cuda.stream(s_h):
                if i >= 2:
                    s_h.wait_event(comp_done[i - 2])        # inputs set b free again
                for k in in_keys:
                    dev_in[b][k].copy_(host_in[k], non_blocking=True)
                h2d_done[i].record(s_h)
            s_c.wait_event(h2d_done[i])
            if i >= 2:
                s_c.wait_event(d2h_done[i - 2])             # outputs set b read out
            d = {k: dev_in[b].get(k, g[k]) for k in ("X", "A", "bias", "B", "dZ")}
            o = {k: dev_out[b].get(k, g[k]) for k in ("Z", "dX", "dA", "dB", "dbias")}
            Z, U, Y = tpl.tp_mlp_fwd(d["X"], d["A"], d["bias"], d["B"], MLP["N"], U=g["U"],
                                     Y=g["Y"], Z=o["Z"], ws=g["ws_f"], dev_status=st)
            tpl.tp_mlp_bwd(d["X"], d["A"], d["B"], U, Y, d["dZ"], MLP["N"], dU=g["dU"],
                           dX=o["dX"], dA=o["dA"], dbias=o["dbias"], dB=o["dB"], ws=g["ws_b"],
                           dev_status=st)
            comp_done[i].record(s_c)
            with torch.cuda.stream(s_d):
                s_d.wait_event(comp_done[i])
                for k in out_keys:
                    host_out[b][k].copy_(dev_out[b][k], non_blocking=True)
                d2h_done[i].record(s_d)
        if timed:
            t1.record(s_d)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / nsteps if timed else None

    run(2, False)
    ms = run(steps, True)
    assert int(st.item()) == 0
    return ms, h2d, d2h


SETTLE_S = 0.1


def _side_loop(torch, fns, plist, nsteps, stream, dev, st, world, reps=10):
    """Average ms per call of each part in plist, max over ranks.

    Each part is captured into a CUDA graph of `reps` back-to-back calls and
    the graph is replayed `nsteps` times between two CUDA events, so host
    launch overhead cannot leave the GPU idle inside the timed interval (it
    would for parts of a few tens of microseconds).  Before its timed
    replays each part replays untimed for at least SETTLE_S seconds: a part
    is then timed at the clocks its own load settles to, not at those the
    previous (power-capped, GEMM-heavy) loop left behind.  Parts that cannot
    be captured are timed as a plain loop of calls instead."""
    for _ in range(2):
        for p in plist:
            fns[p]()
    torch.cuda.synchronize(dev)
    ms = []
    for p in plist:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(reps):
                    fns[p]()
            graph.replay()
            torch.cuda.synchronize(dev)
            t_settle = time.perf_counter()
            while time.perf_counter() - t_settle < SETTLE_S:
                graph.replay()
                torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(nsteps):
                graph.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms.append(e0.elapsed_time(e1) / (nsteps * reps))
            del graph
        except RuntimeError:
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(nsteps):
                fns[p]()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms.append(e0.elapsed_time(e1) / nsteps)
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    t = torch.tensor(ms, dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return {p: float(t[i]) for i, p in enumerate(plist)}


def _event_loop(torch, fn, n, stream, before=None):
    """Average ms of fn() over n calls, each bracketed by its own CUDA events
    on `stream`; before() (untimed) runs ahead of every call."""
    total = 0.0
    evs = []
    for _ in range(n):
        if before is not None:
            before()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    for e0, e1 in evs:
        total += e0.elapsed_time(e1)
    return total / n


def _flushed(torch, fn, dev, stream, n=10):
    """Average ms of fn() with the 126 MB L2 flushed before every call: an
    untimed read of a 256 MB buffer (torch.amax), so that the call's inputs
    come from HBM and no dirty lines of the flush are written back inside
    the timed call (a memset flush would leave 126 MB of them)."""
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    ms = _event_loop(torch, fn, n, stream, before=lambda: torch.amax(flush))
    del flush
    return ms


def _library_context(torch, g, vo, stream, n=10, ours=None):
    """cuBLAS (torch.matmul, bf16 in, fp32 accumulate) on the six GEMM shapes
    of the TP-MLP at h=4096 with the operand transposes the layer needs, and
    torch.nn.functional.cross_entropy (sum, forward + backward) on the same
    fp32 logits as vp_xent.  Library context, not the product's path.
    `ours` (mlp_fwd, mlp_bwd) are timed right after the GEMMs in the same
    kind of loop, so the two sums compare under the same conditions."""
    import torch.nn.functional as F

    X, A, B, dZ, U, Y, dU = (g[k] for k in ("X", "A", "B", "dZ", "U", "Y", "dU"))
    gemms = {
        "a2 U=X·A": lambda: torch.matmul(X, A),
        "a3 Z=Y·B": lambda: torch.matmul(Y, B),
        "a4 dY=dZ·Bt": lambda: torch.matmul(dZ, B.t()),
        "a5 dB=Yt·dZ": lambda: torch.matmul(Y.t(), dZ),
        "a6 dA=Xt·dU": lambda: torch.matmul(X.t(), dU),
        "a7 dX=dU·At": lambda: torch.matmul(dU, A.t()),
    }
    flop = 2.0 * MLP["M"] * MLP["h"] * MLP["F"]
    out = {}
    total = 0.0
    for name, fn in gemms.items():
        for _ in range(3):
            fn()
        ms = _event_loop(torch, fn, n, stream)
        out[name] = {"ms": round(ms, 4), "tflops": round(flop / (ms / 1e3) / 1e12, 1)}
        total += ms
    ctx = {"what": "torch.matmul (cuBLAS) on the six TP-MLP GEMM shapes at h=4096 (no fused "
                   "bias/GeLU/dGeLU, no shard sums), and torch cross_entropy forward+backward on "
                   "the [16384, 50304] fp32 logits; timed in this process after the step, "
                   "%d calls each" % n,
           "mlp_gemms": out, "mlp_gemms_sum_ms": round(total, 4),
           "mlp_gemms_sum_tflops": round(MLP_FLOP / (total / 1e3) / 1e12, 1)}
    if ours is not None:
        fwd, bwd = ours
        for _ in range(3):
            fwd()
            bwd()
        ms_f = _event_loop(torch, fwd, n, stream)
        ms_b = _event_loop(torch, bwd, n, stream)
        ctx["tp_mlp_same_loop"] = {
            "what": "this library's tp_mlp_fwd and tp_mlp_bwd (all six GEMMs with their fused "
                    "bias/GeLU, dGeLU, dbias and shard-sum epilogues) timed the same way, "
                    "%d calls each, right after the cuBLAS GEMMs" % n,
            "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
            "sum_ms": round(ms_f + ms_b, 4),
            "tflops": round(MLP_FLOP / ((ms_f + ms_b) / 1e3) / 1e12, 1),
            "vs_cublas_sum": round(total / (ms_f + ms_b), 4)}
    if vo is not None:
        L = vo["logits"].detach().requires_grad_(True)
        tg = vo["targets"]

        def xent():
            loss = F.cross_entropy(L, tg, reduction="sum")
            loss.backward()
            L.grad = None

        for _ in range(2):
            xent()
        ms = _event_loop(torch, xent, max(3, n // 2), stream)
        ctx["cross_entropy_fwd_bwd_ms"] = round(ms, 4)
        ctx["cross_entropy_tokens_per_s"] = round(VOC["T"] / (ms / 1e3), 1)
    return ctx


def run_gpu(args):
    import torch

    import linear_layers_b200 as tpl
    from linear_layers_b200 import build as tpbuild

    rank, world, local = _dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if rank == 0:
        tpbuild.build()
    if world > 1:
        torch.distributed.barrier()
    tpl.lib()

    known = PARTS + BWD_PARTS[1:] + FUSED_PARTS + RECOMPUTE_PARTS + ATTN_PARTS + LN_PARTS + GEMM_PARTS
    parts = [p for p in known if p in args.parts.split(",")]
    if not parts:
        raise SystemExit(f"--parts must name some of {','.join(known)}")
    if args.vocab_tokens:
        VOC["T"] = args.vocab_tokens
    full = parts == list(PARTS) and VOC["T"] == 16384 and not args.partial
    if full:   # the side loops need their vocabulary buffers too
        parts_prep = parts + list(BWD_PARTS) + list(FUSED_PARTS)
    else:
        parts_prep = parts
    g, pr, vo = _prepare(dev, parts_prep)
    st = tpl.new_status(dev)
    fns = {"mlp_fwd": lambda: _mlp_fwd(tpl, g, st), "mlp_bwd": lambda: _mlp_bwd(tpl, g, st),
           "proj": lambda: _proj(tpl, pr, st), "embed": lambda: _embed(tpl, vo, st),
           "logits": lambda: _logits(tpl, vo, st), "xent": lambda: _xent(tpl, vo, st),
           "xent_bf16": lambda: _xent_bf16(tpl, vo, st),
           "logits_bwd": lambda: _logits_bwd(tpl, vo, st),
           "embed_bwd": lambda: _embed_bwd(tpl, vo, st),
           "lxent_fwd": lambda: _lxent_fwd(tpl, vo, st),
           "lxent_dlogits": lambda: _lxent_dlogits(tpl, vo, st),
           "mlp_bwd_rc": lambda: _mlp_bwd_rc(tpl, g, st),
           "attn_fwd": lambda: _attn_fwd(tpl, pr, st),
           "attn_bwd": lambda: _attn_bwd(tpl, pr, st),
           "ln_fwd": lambda: _ln_fwd(tpl, pr, st),
           "ln_bwd": lambda: _ln_bwd(tpl, pr, st),
           "col_gemm": lambda: _col_gemm(tpl, g, st),
           "cublas_gemm": lambda: _cublas_gemm(torch, g)}
    stream = torch.cuda.current_stream(dev)

    # the clock sampler starts before the warm-up (nvidia-smi takes a moment
    # to write its first sample); mark() keeps the samples of the timed steps
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(args.warmup):
            for p in parts:
                fns[p]()
        torch.cuda.synchronize(dev)
        assert int(st.item()) == 0, f"device status {int(st.item())} after warm-up"

        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)]
              for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        launches0 = tpl.tp_launch_count()
        clk.mark()
        t_wall = time.perf_counter()
        for s in range(args.steps):
            ev[s][0].record(stream)
            for i, p in enumerate(parts):
                fns[p]()
                ev[s][i + 1].record(stream)
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall
    launches = tpl.tp_launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    assert int(st.item()) == 0, f"device status {int(st.item())}"

    part_ms = {p: 0.0 for p in parts}
    total_ms = 0.0
    for s in range(args.steps):
        total_ms += ev[s][0].elapsed_time(ev[s][-1])
        for i, p in enumerate(parts):
            part_ms[p] += ev[s][i].elapsed_time(ev[s][i + 1])
    times = torch.tensor([total_ms] + [part_ms[p] for p in parts], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(times, op=torch.distributed.ReduceOp.MAX)
    total_ms = float(times[0])
    part_ms = {p: float(times[i + 1]) for i, p in enumerate(parts)}
    if not full:   # a partial run (profiling): report the part times only
        graphed = _side_loop(torch, fns, parts, max(args.steps, 5), stream, dev, st, world)
        if rank == 0:
            print(json.dumps({"partial_run": True, "parts": parts, "vocab_tokens": VOC["T"],
                              "steps": args.steps, "warmup": args.warmup,
                              "parts_ms_per_step": {p: round(part_ms[p] / args.steps, 4)
                                                    for p in parts},
                              "parts_ms_graph_replay": {p: round(graphed[p], 4) for p in parts},
                              "gpu_launches": int(launches)}), flush=True)
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return

    # vocabulary backward and the fused output layer + loss: their own timed
    # loops (not part of the step)
    side_steps = max(5, min(args.steps, 20))
    bwd_ms = _side_loop(torch, fns, BWD_PARTS, side_steps, stream, dev, st, world)
    fused_ms = _side_loop(torch, fns, FUSED_PARTS, side_steps, stream, dev, st, world)
    rc_ms = _side_loop(torch, fns, RECOMPUTE_PARTS, side_steps, stream, dev, st, world)
    at_ms = _side_loop(torch, fns, ATTN_PARTS, side_steps, stream, dev, st, world)
    ln_ms = _side_loop(torch, fns, LN_PARTS, side_steps, stream, dev, st, world)

    embed_flush_ms = _flushed(torch, fns["embed"], dev, stream)
    ln_flush_ms = {p: _flushed(torch, fns[p], dev, stream) for p in LN_PARTS}
    libctx = (None if args.no_library_context else
              _library_context(torch, g, vo, stream, ours=(fns["mlp_fwd"], fns["mlp_bwd"])))

    if args.no_e2e:
        e2e_ms, h2d, d2h = float("nan"), 0, 0
        all_ms, all_h2d, all_d2h = float("nan"), 0, 0
    else:
        e2e_ms, h2d, d2h = _e2e_mlp(tpl, torch, g, dev, max(4, min(args.steps, 8)))
        all_ms, all_h2d, all_d2h = _e2e_mlp(tpl, torch, g, dev, max(4, min(args.steps, 8)), E2E_ALL)
    e2e = torch.tensor([e2e_ms, all_ms], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(e2e, op=torch.distributed.ReduceOp.MAX)
    e2e_ms, all_ms = float(e2e[0]), float(e2e[1])
    clocks = clk.summary()

    if rank == 0:
        peaks, src = _peaks()
        K = args.steps
        mlp_s = (part_ms["mlp_fwd"] + part_ms["mlp_bwd"]) / 1e3
        value = world * K * MLP_FLOP / mlp_s / 1e12
        xent_s = part_ms["xent"] / 1e3
        tok_s = world * K * VOC["T"] / xent_s
        xent_gbs = K * XENT_BYTES / xent_s / 1e9
        embed_gbs = K * EMBED_BYTES / (part_ms["embed"] / 1e3) / 1e9
        gemm_flop = K * (MLP_FLOP + PROJ_FLOP + LOGITS_FLOP)
        gemm_s = (part_ms["mlp_fwd"] + part_ms["mlp_bwd"] + part_ms["proj"] + part_ms["logits"]) / 1e3
        achieved = gemm_flop / gemm_s / 1e12
        peak = peaks["bf16_tflops_sustained"]
        traffic, traffic_note = _roofline_traffic()
        out = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(total_ms / K, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic: seeded N(0,sigma) activations and random-init weights, uniform token ids",
            "config": {
                "workload": "tp_mlp M=4096 h=4096 ffn=16384 N=8 fwd+bwd; gpt2-1.5B slice attention "
                            "projections M=4096 h=1600 heads 7/6/6/6; vocab T=16384 v=50304 N=8 h=4096 "
                            "embed+logits+xent",
                "global_batch": MLP["M"],
                "seq_len": 2048,
                "parallelism": f"tp{MLP['N']} logical shards on one GPU; {world} replica(s)",
                "l2": "inputs larger than L2 (>= 4 GB touched per step vs 126 MB L2); no flush",
            },
            "mlp_fwd_bwd": {"tflops": round(value / world, 2), "frac_of_spec_2250": round(value / world / SPEC_BF16_TFLOPS, 4),
                            "frac_of_measured_burst": round(value / world / peaks["bf16_tflops"], 4),
                            "ms": round(mlp_s * 1e3 / K, 4)},
            "vocab_xent": {"tokens_per_s": round(tok_s, 1), "GBps": round(xent_gbs, 1),
                           "frac_of_measured_hbm": round(xent_gbs / peaks["hbm_gbs"], 4),
                           "frac_of_spec_8000": round(xent_gbs / SPEC_HBM_GBS, 4),
                           "ms": round(part_ms["xent"] / K, 4)},
            "vp_embed": {"GBps": round(embed_gbs, 1), "frac_of_measured_hbm": round(embed_gbs / peaks["hbm_gbs"], 4),
                         "us": round(part_ms["embed"] / K * 1e3, 2),
                         "l2_flushed": {"us": round(embed_flush_ms * 1e3, 2),
                                        "GBps": round(EMBED_BYTES / (embed_flush_ms / 1e3) / 1e9, 1),
                                        "frac_of_measured_hbm": round(EMBED_BYTES / (embed_flush_ms / 1e3) / 1e9
                                                                      / peaks["hbm_gbs"], 4),
                                        "what": "a 256 MB read before every call (untimed), 10 calls"}},
            "vocab_bwd": {
                "what": "next row, own loop of %d iterations after the step" % side_steps,
                "xent_bf16_grad_ms": round(bwd_ms["xent_bf16"], 4),
                "xent_bf16_grad_GBps": round(XENT_BF16_BYTES / (bwd_ms["xent_bf16"] / 1e3) / 1e9, 1),
                "logits_bwd_ms": round(bwd_ms["logits_bwd"], 4),
                "logits_bwd_tflops": round(LOGITS_BWD_FLOP / (bwd_ms["logits_bwd"] / 1e3) / 1e12, 1),
                "embed_bwd_us": round(bwd_ms["embed_bwd"] * 1e3, 1),
            },
            "linear_xent": {
                "what": "output layer + loss without the [T,v] logits: statistics GEMM + combine "
                        "(loss, lse, argmax), then the recomputing bf16-gradient GEMM; own loop of "
                        "%d iterations" % side_steps,
                "fwd_ms": round(fused_ms["lxent_fwd"], 4),
                "fwd_tflops": round(LOGITS_FLOP / (fused_ms["lxent_fwd"] / 1e3) / 1e12, 1),
                "unfused_logits_plus_xent_ms": round((part_ms["logits"] + part_ms["xent"]) / K, 4),
                "dlogits_ms": round(fused_ms["lxent_dlogits"], 4),
                "dlogits_tflops": round(LOGITS_FLOP / (fused_ms["lxent_dlogits"] / 1e3) / 1e12, 1),
                "logits_bytes_not_stored": VOC["T"] * VOC["v"] * 4,
            },
            "mlp_bwd_recompute": {
                "what": "TP-MLP backward from the saved pre-activation U alone (Y = GeLU(U) rebuilt "
                        "in the dGeLU GEMM's epilogue); own loop of %d iterations" % side_steps,
                "ms": round(rc_ms["mlp_bwd_rc"], 4),
                "tflops": round(4.0 * MLP["M"] * MLP["h"] * MLP["F"] * 2 / (rc_ms["mlp_bwd_rc"] / 1e3) / 1e12, 1),
                "saved_activation_ms": round(part_ms["mlp_bwd"] / K, 4),
                "activation_bytes_not_kept": MLP["M"] * MLP["F"] * 2,
            },
            "attention_fwd": {
                "what": "causal attention core between the projections, b=4 s=1024, 25 heads of 64 "
                        "over 4 shards (7/6/6/6); own loop of %d iterations" % side_steps,
                "us": round(at_ms["attn_fwd"] * 1e3, 2),
                "tflops": round(ATTN_FLOP / (at_ms["attn_fwd"] / 1e3) / 1e12, 1),
                "bwd_us": round(at_ms["attn_bwd"] * 1e3, 2),
                "bwd_tflops": round(2.5 * ATTN_FLOP / (at_ms["attn_bwd"] / 1e3) / 1e12, 1),
                "bwd_flop_note": "2.5x the forward's: Sᵀ, dPᵀ, dV, dK in one kernel and S, dP, dQ "
                                 "in the other (7 products of which 5 are the algorithmic ones)",
                "flop_note": "4·b·heads·d·s(s+1)/2 (the unmasked half of Q·Kᵀ and P·V)",
            },
            "sp_layernorm": {
                "what": "hs = X + dropout(Zo + b), y = LayerNorm(hs) and its backward, M=4096 "
                        "h=1600 over 4 sequence shards, p=0.1 (Philox masks regenerated in the "
                        "backward); own loop of %d iterations: its 52-65 MB working set stays in "
                        "the 126 MB L2 between calls, so these are L2-warm; l2_flushed has the "
                        "HBM-bound figures" % side_steps,
                "fwd_us": round(ln_ms["ln_fwd"] * 1e3, 2),
                "fwd_GBps": round(LN_FWD_BYTES / (ln_ms["ln_fwd"] / 1e3) / 1e9, 1),
                "bwd_us": round(ln_ms["ln_bwd"] * 1e3, 2),
                "bwd_GBps": round(LN_BWD_BYTES / (ln_ms["ln_bwd"] / 1e3) / 1e9, 1),
                "l2_flushed": {
                    "what": "a 256 MB read before every call (untimed), 10 calls each",
                    "fwd_us": round(ln_flush_ms["ln_fwd"] * 1e3, 2),
                    "fwd_GBps": round(LN_FWD_BYTES / (ln_flush_ms["ln_fwd"] / 1e3) / 1e9, 1),
                    "fwd_frac_of_measured_hbm": round(LN_FWD_BYTES / (ln_flush_ms["ln_fwd"] / 1e3) / 1e9
                                                      / peaks["hbm_gbs"], 4),
                    "bwd_us": round(ln_flush_ms["ln_bwd"] * 1e3, 2),
                    "bwd_GBps": round(LN_BWD_BYTES / (ln_flush_ms["ln_bwd"] / 1e3) / 1e9, 1),
                    "bwd_frac_of_measured_hbm": round(LN_BWD_BYTES / (ln_flush_ms["ln_bwd"] / 1e3) / 1e9
                                                      / peaks["hbm_gbs"], 4),
                },
                "bytes_note": "8 B/element forward (x, residual in; hs, y out), 10 B/element "
                              "backward (dy, dhs, hs in; dx, dresidual out)",
            },
            "parts_ms_per_step": {p: round(part_ms[p] / K, 4) for p in PARTS},
            "roofline": {
                "kernel": "gemm_tc_kernel (all 13 GEMM launches of the step)",
                "bound": "tensor",
                "achieved": round(achieved, 2),
                "peak": peak,
                "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "peak_source": f"{src} bf16_tflops_sustained (kernel timed inside a long step)",
                "traffic": traffic,
                "traffic_unit": "bytes/launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                "traffic_note": traffic_note,
            },
            "library_context": libctx,
            "gpu_launches": int(launches),
            "clocks": clocks,
            "wall_s_timed": round(t_wall, 3),
            "e2e": {"value": round(world * MLP_FLOP / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "what": "tp_mlp_fwd+tp_mlp_bwd through the public API; every step copies its data "
                            "(X, dZ) from pinned host memory and reads its results (Z, dX) back inside "
                            "the timed region; weights and weight gradients stay resident on the device "
                            "as in a training loop; copies of neighbouring steps overlap the compute on "
                            "their own streams; timed in its own TP-MLP-only loop after the step (the "
                            "step's other parts do not run between its iterations), so it is not measured "
                            "under the same conditions as value",
                    "all_tensors": {"value": round(world * MLP_FLOP / (all_ms / 1e3) / 1e12, 2),
                                    "h2d_bytes_per_step": int(all_h2d),
                                    "d2h_bytes_per_step": int(all_d2h),
                                    "what": "the same with the weights copied in and the weight "
                                            "gradients read back every step as well"}},
        }
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ----------------------------------------------------------------------------
# the oracle on the host (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _oracle_mlp_sample(rows: int):
    """fp64 oracle forward + backward of the TP-MLP on `rows` token rows of the
    M=4096, h=4096, ffn=16384 layer.  Returns (seconds, flops)."""
    import tp_inputs
    from oracle import tp_oracle as O

    inp = tp_inputs.mlp_inputs(rows, MLP["h"], MLP["F"], w_std=MLP["w_std"], seed=0)
    t0 = time.perf_counter()
    O.mlp_fwd(inp["X"], inp["A"], inp["bias"], inp["B"])
    O.mlp_bwd(inp["X"], inp["A"], inp["bias"], inp["B"], inp["dZ"])
    dt = time.perf_counter() - t0
    # the oracle's backward recomputes the forward: count the layer's 6 GEMMs once
    return dt, 12.0 * rows * MLP["h"] * MLP["F"]


def cpu_baseline(budget_s: float = 15.0):
    rows = 64
    dt, fl = _oracle_mlp_sample(rows)
    # grow the sample toward the time budget (bounded by the layer's 4096 rows);
    # the small first samples carry fixed costs, so the growth is taken twice
    for _ in range(2):
        if dt >= budget_s / 2 or rows >= MLP["M"]:
            break
        rows = int(min(MLP["M"], max(64, rows * 0.8 * budget_s / max(dt, 1e-3))))
        rows = max(64, rows // 64 * 64)
        dt, fl = _oracle_mlp_sample(rows)
    return {"value": round(fl / dt / 1e12, 5), "unit": "TFLOP/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle, TP-MLP fwd+bwd on {rows} of 4096 token rows "
                      f"(h=4096, ffn=16384), {dt:.1f} s; cpu={os.cpu_count()} logical"}


def run_reference(args):
    rank, world, _ = _dist_env()
    if rank != 0:
        return
    rows = args.ref_rows
    _oracle_mlp_sample(rows)   # warm-up (also pages in BLAS)
    total_t, total_f = 0.0, 0.0
    for _ in range(args.warmup):
        _oracle_mlp_sample(rows)
    for _ in range(args.steps):
        dt, fl = _oracle_mlp_sample(rows)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    cores = _blas_threads()
    sample = (f"fp64 numpy oracle, TP-MLP fwd+bwd on {rows} of 4096 token rows (h=4096, ffn=16384) "
              f"per step; cpu={os.cpu_count()} logical")
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 5),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_t / args.steps * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: seeded N(0,sigma) activations and random-init weights",
        "config": {"workload": "tp_mlp M=4096 h=4096 ffn=16384 N=8 fwd+bwd (row sample)",
                   "global_batch": MLP["M"], "seq_len": 2048, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--parts", default=",".join(PARTS),
                    help="comma-separated subset of the step (profiling runs); the JSON line of "
                         "a partial run only carries part times")
    ap.add_argument("--vocab-tokens", type=int, default=0,
                    help="tokens of the vocabulary path (profiling runs; default 16384)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-library-context", action="store_true")
    ap.add_argument("--partial", action="store_true",
                    help="report part times only, also for the whole step (sweeps)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps, always
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
