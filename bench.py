"""Benchmark of the fused RHT + group-quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {hit,reference}]
                    [--workload weight_rht_int4|activation_rht|activation_quant|two_sided_lowbit|wht_adapter|
                                two_sided_butterfly|mixed_rht_int4|harp_rotation]
                    [--bits 2|3]   (two_sided_lowbit only)

Default workload (the headline metric): fp32 4096 x 4096 weights, row RHT
(n = 4096, Rademacher signs) fused with symmetric absmax 4-bit RTN in groups
of 128 and nibble packing, one rht_quantize_pack launch per step.  Inputs are
resident in HBM; each step uses the next of R rotating input/output buffer
sets whose total exceeds 4x the L2 size, so no step reads its input from L2.
Throughput counts algorithmic bytes only (input read once, codes and scales
written once).  Prints one JSON line (rank 0).

--impl reference times the CPU oracle (the reference arm) on a
bounded sample of the same workload per step.

--gpus N without torchrun re-launches this script under torch.distributed.run
with N ranks (one per GPU); under torchrun, --gpus must equal WORLD_SIZE.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "fused RHT+group-quant effective HBM GB/s and % of peak; rows/s at d=4096"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------
# multi-rank plumbing
# ----------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        import datetime

        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def reduce_max(value: float, dist, device) -> float:
    """Max of a per-rank float over all ranks (identity on one rank)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ----------------------------------------------------------------------------
# measurement helpers
# ----------------------------------------------------------------------------
def measured_peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[index]) if vis and vis.split(",")[index].isdigit() else index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            time.sleep(0.0002)  # the headline's timed region is only ~8 ms long

    def __enter__(self):
        self.t_begin = time.perf_counter()
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            # the sampler is running before the timed region starts
            t0 = time.perf_counter()
            while len(self.samples) < 2 and time.perf_counter() - t0 < 0.5:
                time.sleep(0.0005)
        self.t_begin = time.perf_counter()
        return self

    def __exit__(self, *exc):
        self.t_end = time.perf_counter()
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        """Samples taken while the timed region ran (host window around it);
        the last earlier sample if none fell inside."""
        inside = [s for s in self.samples if self.t_begin <= s[0] <= getattr(self, "t_end", float("inf"))]
        used = inside or self.samples[-1:]
        reasons = set()
        for _, _, r in used:
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    reasons.add(name)
        med = statistics.median(m for _, m, _ in used) if used else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(inside)}


def read_profile_traffic(kernel_key: str):
    """Per-launch DRAM bytes of `kernel_key` from profiles/traffic.json, if the
    digest of the sources the record names (the kernel's translation unit and
    the build script) still matches (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_key)
        if rec and rec.get("source_digest") == source_digest(rec["sources"]):
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def source_digest(sources) -> str:
    """sha256 prefix over the named files (paths relative to the package directory)."""
    import hashlib

    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "hadamard_incoherence_transforms_b200")
    for rel in sources:
        with open(os.path.join(pkg, rel), "rb") as fh:
            h.update(rel.encode() + fh.read())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------
# workloads: build device buffers and a step function
# ----------------------------------------------------------------------------
class Workload:
    """name, algorithmic bytes and rows per step, a step(i) launching the GPU
    hot path on rotation set i, host-buffer e2e step, and an oracle sample.
    `dtype` is the arithmetic type of the path (fp32 registers for the SIMT
    kernels whatever the storage type; bf16 operands with fp32 accumulation
    on the tensor cores)."""

    dtype = "f32"


def _quant_parity(codes_rows, scales_rows, ref, bits, n) -> dict:
    """Codes and scales of sampled rows against the oracle's: codes differing
    outside the rounding-boundary window (must be 0), excused ones, and the
    largest relative scale error."""
    from oracle import quant as oq

    u = oq.unpack(codes_rows.cpu().numpy(), bits, n)
    diff = u != ref["u"]
    win = oq.boundary_window(ref["t"])
    s = scales_rows.cpu().numpy().astype(np.float64)
    rs = ref["scales"].astype(np.float64)
    rel = np.abs(s - rs) / np.where(rs > 0, rs, 1.0)
    return {"rows": int(u.shape[0]), "codes_outside_window": int((diff & ~win).sum()),
            "codes_excused": int((diff & win).sum()), "codes": int(u.size),
            "scale_rel_max": float(rel.max(initial=0.0))}


def _rel_l2(got, ref) -> float:
    ref = np.asarray(ref, np.float64)
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(np.asarray(got, np.float64) - ref) / (den if den > 0 else 1.0))


def _bf16_row_rel(got, ref) -> float:
    ref = np.asarray(ref, np.float64)
    d = np.abs(np.asarray(got, np.float64) - ref).max(axis=-1)
    m = np.abs(ref).max(axis=-1)
    return float((d / np.where(m > 0, m, 1.0)).max())


def _host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def weight_rht_int4(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.weight_rht_int4()
    rows, n, bits, group = 4096, 4096, 4, 128
    in_b = rows * n * 4
    out_b = rows * n * bits // 8 + rows * (n // group) * 4
    w = Workload()
    w.name = "weight_rht_int4"
    w.desc = "fp32 4096x4096 N(0,0.02) + 0.1% outliers x50; row RHT n=4096 + 4-bit absmax RTN g=128, packed"
    w.io = "fp32 in; 4-bit codes + fp32 scales out"
    w.rows, w.n, w.bytes = rows, n, in_b + out_b
    w.h2d, w.d2h = in_b, out_b
    w.data = d
    w.kernels_per_step = 1
    w.kernel_key = "k_rows_stream<12,float,float,EPI_QUANT,4>"

    def oracle(r0, r1):
        from oracle import hadamard as oh
        from oracle import quant as oq

        q = oq.quantize(oh.rht_rows(d["x"][r0:r1], d["signs"]), bits, group)
        oq.pack(q["u"], bits)
        return q

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    R = max(2, math.ceil(4 * l2_bytes / (in_b + out_b)) + 1)
    x0 = torch.from_numpy(d["x"]).to(dev)
    xs = [x0] + [x0.clone() for _ in range(R - 1)]
    s = torch.from_numpy(d["signs"]).to(dev)
    cs = [torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8, device=dev) for _ in range(R)]
    ss = [torch.empty((rows, n // group), dtype=torch.float32, device=dev) for _ in range(R)]
    w.rotation = R

    def step(i):
        k = i % R
        hit.rht_quantize_pack(xs[k], s, bits, group, codes=cs[k], scales=ss[k])

    w.step = step
    w.parity = lambda ref, r0, r1: _quant_parity(cs[0][r0:r1], ss[0][r0:r1], ref, bits, n)
    hx = torch.from_numpy(d["x"]).pin_memory()
    hc = torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8).pin_memory()
    hs = torch.empty((rows, n // group), dtype=torch.float32).pin_memory()

    def e2e_step(i):
        k = i % R
        xs[k].copy_(hx, non_blocking=True)
        hit.rht_quantize_pack(xs[k], s, bits, group, codes=cs[k], scales=ss[k])
        hc.copy_(cs[k], non_blocking=True)
        hs.copy_(ss[k], non_blocking=True)

    w.e2e_step = e2e_step
    return w


def activation_rht(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.activation_rht()
    rows, n = 8192, 4096
    w = Workload()
    w.name, w.rows, w.n = "activation_rht", rows, n
    w.desc = "bf16 8192x4096 0.5*t3 + 1% columns x20; row RHT n=4096, bf16 in/out, fp32 accumulate"
    w.io = "bf16 in; bf16 out"
    w.bytes = rows * n * 4
    w.h2d = w.d2h = rows * n * 2
    w.kernels_per_step = 1
    w.kernel_key = "k_rows_stream<12,bf16,bf16,EPI_STORE,0>"

    def oracle(r0, r1):
        from oracle import hadamard as oh

        return oh.rht_rows(synth.bf16_bits_to_f32(d["x_bf16"][r0:r1]), d["signs"])

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    R = max(2, math.ceil(4 * l2_bytes / w.bytes) + 1)
    x0 = torch.from_numpy(d["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    xs = [x0] + [x0.clone() for _ in range(R - 1)]
    ys = [torch.empty_like(x0) for _ in range(R)]
    s = torch.from_numpy(d["signs"]).to(dev)
    w.rotation = R
    w.step = lambda i: hit.rht_forward(xs[i % R], s, out=ys[i % R])
    w.parity = lambda ref, r0, r1: {"rows": r1 - r0, "bf16_row_rel_max": _bf16_row_rel(_host64(ys[0][r0:r1]), ref)}
    hx = x0.cpu().pin_memory()
    hy = torch.empty_like(hx).pin_memory()

    def e2e_step(i):
        k = i % R
        xs[k].copy_(hx, non_blocking=True)
        hit.rht_forward(xs[k], s, out=ys[k])
        hy.copy_(ys[k], non_blocking=True)

    w.e2e_step = e2e_step
    return w


def activation_quant(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.activation_rht()
    rows, n, bits, group = 8192, 4096, 4, 4096
    w = Workload()
    w.name, w.rows, w.n = "activation_quant", rows, n
    w.desc = "bf16 8192x4096 0.5*t3 + 1% columns x20; row RHT n=4096 + 4-bit absmax RTN, one scale per token"
    w.io = "bf16 in; 4-bit codes + fp32 per-token scales out"
    in_b = rows * n * 2
    out_b = rows * n * bits // 8 + rows * 4
    w.bytes = in_b + out_b
    w.h2d, w.d2h = in_b, out_b
    w.kernels_per_step = 1
    w.kernel_key = "k_rows_stream<12,bf16,float,EPI_QUANT,4>"
    xb = synth.bf16_bits_to_f32(d["x_bf16"])

    def oracle(r0, r1):
        from oracle import hadamard as oh
        from oracle import quant as oq

        q = oq.quantize(oh.rht_rows(xb[r0:r1], d["signs"]), bits, group)
        oq.pack(q["u"], bits)
        return q

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    R = max(2, math.ceil(4 * l2_bytes / w.bytes) + 1)
    x0 = torch.from_numpy(d["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    xs = [x0] + [x0.clone() for _ in range(R - 1)]
    s = torch.from_numpy(d["signs"]).to(dev)
    cs = [torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8, device=dev) for _ in range(R)]
    ss = [torch.empty((rows, 1), dtype=torch.float32, device=dev) for _ in range(R)]
    w.rotation = R

    def step(i):
        k = i % R
        hit.rht_quantize_pack(xs[k], s, bits, group, codes=cs[k], scales=ss[k])

    w.step = step
    w.parity = lambda ref, r0, r1: _quant_parity(cs[0][r0:r1], ss[0][r0:r1], ref, bits, n)
    hx = x0.cpu().pin_memory()
    hc = torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8).pin_memory()
    hs = torch.empty((rows, 1), dtype=torch.float32).pin_memory()

    def e2e_step(i):
        k = i % R
        xs[k].copy_(hx, non_blocking=True)
        hit.rht_quantize_pack(xs[k], s, bits, group, codes=cs[k], scales=ss[k])
        hc.copy_(cs[k], non_blocking=True)
        hs.copy_(ss[k], non_blocking=True)

    w.e2e_step = e2e_step
    return w


def two_sided_lowbit(dev, l2_bytes, host_only=False, bits=3, **_):
    import synth

    d = synth.two_sided_lowbit()
    rows = n = 8192
    group = 64
    w = Workload()
    w.name, w.rows, w.n = f"two_sided_lowbit_{bits}b", rows, n
    w.desc = f"bf16 8192x8192 + 0.05% outliers x100; two-sided RHT + {bits}-bit g=64 then dequant + inverse (fp32 out)"
    w.io = f"bf16 in; {bits}-bit codes + fp32 scales; fp32 reconstruction out"
    q_b = rows * n * bits // 8 + rows * (n // group) * 4
    w.bytes = rows * n * 2 + q_b + q_b + rows * n * 4
    w.h2d, w.d2h = rows * n * 2, rows * n * 4
    w.kernels_per_step = 4  # column pass + row quantize; row dequantize + column pass
    w.kernel_key = "k_cols_cluster<8,bf16,float>"
    xb = synth.bf16_bits_to_f32(d["x_bf16"])  # the bf16 input widened once (input preparation)

    def oracle(r0, r1):
        from oracle import hadamard as oh
        from oracle import quant as oq

        idx = np.arange(r0, r1)
        return oq.quantize(oh.two_sided_rows_at(xb, d["row_signs"], d["col_signs"], idx), bits, group)

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    x = torch.from_numpy(d["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    rs = torch.from_numpy(d["row_signs"]).to(dev)
    cs = torch.from_numpy(d["col_signs"]).to(dev)
    ws = torch.empty(rows * n, dtype=torch.float32, device=dev)
    codes = torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, n // group), dtype=torch.float32, device=dev)
    y = torch.empty((rows, n), dtype=torch.float32, device=dev)
    w.rotation = 1

    def step(i):
        hit.rht_quantize_pack(x, rs, bits, group, col_signs=cs, codes=codes, scales=scales, workspace=ws)
        hit.dequant_inverse(codes, scales, n, bits, group, rs, col_signs=cs, out=y)

    w.step = step
    w.parity = lambda ref, r0, r1: _quant_parity(codes[r0:r1], scales[r0:r1], ref, bits, n)

    def extra():
        """Reconstruction MSE of the timed outputs (float64 on the device) next
        to the oracle's own round-trip MSE (tests/golden, written by the oracle)."""
        mse = float(((y.double() - x.double()) ** 2).mean().item())
        try:
            with open(os.path.join(ROOT, "tests", "golden", "two_sided_lowbit_mse.json")) as f:
                mse_oracle = float(json.load(f)["mse"][str(bits)])
        except Exception:
            mse_oracle = None
        rel = None if not mse_oracle else abs(mse - mse_oracle) / mse_oracle
        return {"mse": mse, "mse_oracle": mse_oracle, "mse_rel_diff": rel}

    w.extra = extra
    hx = x.cpu().pin_memory()
    hy = torch.empty((rows, n), dtype=torch.float32).pin_memory()

    def e2e_step(i):
        x.copy_(hx, non_blocking=True)
        step(i)
        hy.copy_(y, non_blocking=True)

    w.e2e_step = e2e_step
    return w


def wht_adapter(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.wht_adapter()
    bsz, rows, n, nnz = 32, 4096, 4096, 64
    w = Workload()
    w.name, w.rows, w.n = "wht_adapter", bsz * rows, n
    w.desc = "32 x 4096 x 4096 sparse F (64 nnz/row) -> dense dW = F H/64 (fwd) and grad gather (bwd)"
    w.io = "fp32 values + int32 columns in; fp32 dense out (fwd); fp32 dense in, fp32 values out (bwd)"
    w.bytes = 2 * (bsz * rows * nnz * 8 + bsz * rows * n * 4)
    w.h2d, w.d2h = bsz * rows * nnz * 8, bsz * rows * nnz * 4
    w.kernels_per_step = 2
    w.kernel_key = "k_rows_b2a<12,float,PRO_SCATTER,0>"

    def oracle(r0, r1):
        # both directions, like the step: expansion of the rows' coefficients,
        # then the gradient gather from that dense block; flat row r is row
        # r % rows of matrix r // rows
        from oracle import sparse as osp

        dense, grad = [], []
        r = r0
        while r < r1:
            b, a0 = divmod(r, rows)
            a1 = min(rows, a0 + (r1 - r))
            dn = osp.expand(d["values"][b:b + 1, a0:a1], d["cols"][b:b + 1, a0:a1], n, 1 / 64)
            dense.append(dn)
            grad.append(osp.gather_grad(dn, d["cols"][b:b + 1, a0:a1], 1 / 64))
            r += a1 - a0
        return np.concatenate(dense, axis=1), np.concatenate(grad, axis=1)

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    v = torch.from_numpy(d["values"]).to(dev)
    c = torch.from_numpy(d["cols"]).to(dev)
    g = torch.empty_like(v)
    dense = torch.empty((bsz, rows, n), dtype=torch.float32, device=dev)
    w.rotation = 1

    def step(i):
        hit.wht_expand(v, c, n, 1 / 64, out=dense)
        hit.wht_gather(dense, c, 1 / 64, out=g)

    w.step = step
    w.parity = lambda ref, r0, r1: {"rows": r1 - r0, "dense_rel_l2": _rel_l2(_host64(dense[:1, r0:r1]), ref[0]),
                                    "grad_rel_l2": _rel_l2(_host64(g[:1, r0:r1]), ref[1])}
    hv = v.cpu().pin_memory()
    hg = torch.empty_like(hv).pin_memory()

    def e2e_step(i):
        v.copy_(hv, non_blocking=True)
        step(i)
        hg.copy_(g, non_blocking=True)

    w.e2e_step = e2e_step
    return w


def two_sided_butterfly(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.two_sided_butterfly()
    rows, n = 4096, 14336
    w = Workload()
    w.name, w.rows, w.n = "two_sided_butterfly", rows, n
    w.desc = ("bf16 4096x14336: R_in (7,16,16,8) along rows then R_out (16,16,16) along columns, "
              "tensor-core window products (bf16 operands, fp32 accumulation), bf16 between passes")
    w.io = "bf16 in; bf16 out"
    w.dtype = "bf16"
    w.bytes = rows * n * 4
    w.h2d = w.d2h = rows * n * 2
    # R_in: strided two-digit pass, compose + tcgen05 row pass; R_out: two
    # compose + tcgen05 column passes
    w.kernels_per_step = 7
    w.kernel_key = "k_bfly_strided"

    def oracle(r0, r1):
        from oracle import butterfly as ob

        return ob.apply_stages(synth.bf16_bits_to_f32(d["x_bf16"][r0:r1]), d["radices_in"], d["blocks_in"])

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    x = torch.from_numpy(d["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    bi = [torch.from_numpy(b).to(dev) for b in d["blocks_in"]]
    bo = [torch.from_numpy(b).to(dev) for b in d["blocks_out"]]
    mid = torch.empty((rows, n), dtype=torch.bfloat16, device=dev)
    y = torch.empty_like(x)
    wsi = torch.empty(hit.butterfly_tc_workspace_bytes(rows, n, d["radices_in"], 1) // 4 + 64, device=dev)
    wso = torch.empty(hit.butterfly_tc_workspace_bytes(rows, n, d["radices_out"], 0) // 4 + 64, device=dev)
    w.rotation = 1

    def step(i):
        hit.butterfly_apply_tc(x, d["radices_in"], bi, axis=1, out=mid, workspace=wsi)
        hit.butterfly_apply_tc(mid, d["radices_out"], bo, axis=0, out=y, workspace=wso)

    w.step = step
    # the row side (R_in) of the sampled rows, as held (bf16) between the two sides
    w.parity = lambda ref, r0, r1: {"rows": r1 - r0, "row_side_bf16_row_rel": _bf16_row_rel(_host64(mid[r0:r1]), ref)}
    hx = x.cpu().pin_memory()
    hy = torch.empty_like(hx).pin_memory()

    def e2e_step(i):
        x.copy_(hx, non_blocking=True)
        step(i)
        hy.copy_(y, non_blocking=True)

    w.e2e_step = e2e_step
    return w


def mixed_rht_int4(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.mixed_rht_int4()
    rows, n, bits, group = 4096, 5120, 4, 128
    w = Workload()
    w.name, w.rows, w.n = "mixed_rht_int4", rows, n
    w.desc = ("fp32 4096x5120 N(0,0.02) + 0.1% outliers x50; mixed-radix RHT (8,8,8,5,2), QR mixer for radix 5, "
              "+ 4-bit absmax RTN g=128, packed")
    w.io = "fp32 in; 4-bit codes + fp32 scales out"
    in_b = rows * n * 4
    out_b = rows * n * bits // 8 + rows * (n // group) * 4
    w.bytes = in_b + out_b
    w.h2d, w.d2h = in_b, out_b
    w.kernels_per_step = 1
    w.kernel_key = "k_rows_mixed5120_q4"
    g5 = d["mixers"][5][0]

    def oracle(r0, r1):
        from oracle import butterfly as ob
        from oracle import quant as oq

        blocks = ob.rht_stage_blocks(d["radices"], d["mixers"])
        q = oq.quantize(ob.rht_mixed(d["x"][r0:r1], d["signs"], d["radices"], blocks), bits, group)
        oq.pack(q["u"], bits)
        return q

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    R = max(2, math.ceil(4 * l2_bytes / w.bytes) + 1)
    x0 = torch.from_numpy(d["x"]).to(dev)
    xs = [x0] + [x0.clone() for _ in range(R - 1)]
    s = torch.from_numpy(d["signs"]).to(dev)
    cs = [torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8, device=dev) for _ in range(R)]
    ss = [torch.empty((rows, n // group), dtype=torch.float32, device=dev) for _ in range(R)]
    w.rotation = R

    def step(i):
        k = i % R
        hit.rht_mixed_quantize_pack(xs[k], s, g5, codes=cs[k], scales=ss[k])

    w.step = step
    w.parity = lambda ref, r0, r1: _quant_parity(cs[0][r0:r1], ss[0][r0:r1], ref, bits, n)
    hx = torch.from_numpy(d["x"]).pin_memory()
    hc = torch.empty(hit.codes_shape(rows, n, bits), dtype=torch.uint8).pin_memory()
    hs = torch.empty((rows, n // group), dtype=torch.float32).pin_memory()

    def e2e_step(i):
        k = i % R
        xs[k].copy_(hx, non_blocking=True)
        hit.rht_mixed_quantize_pack(xs[k], s, g5, codes=cs[k], scales=ss[k])
        hc.copy_(cs[k], non_blocking=True)
        hs.copy_(ss[k], non_blocking=True)

    w.e2e_step = e2e_step
    return w


def harp_rotation(dev, l2_bytes, host_only=False, **_):
    import synth

    d = synth.harp_rotation()
    rows, n = 4096, 4096
    radices = d["radices"]
    w = Workload()
    w.name, w.rows, w.n = "harp_rotation", rows, n
    w.desc = ("fp32 4096x4096 weights; HARP blocks Q(theta) G_16 built on the device for radices (16,16,16) "
              "(Cayley, theta ~ N(0,0.05)), signs folded into stage 0, then y = R(theta) diag(s) x")
    w.io = "fp32 in; fp32 out"
    w.bytes = rows * n * 8
    w.h2d = w.d2h = rows * n * 4
    w.kernels_per_step = 3 + 2  # three block builds, two butterfly passes
    w.kernel_key = "k_bfly_pass"

    def oracle(r0, r1):
        from oracle import harp as oha

        return oha.forward(d["x"][r0:r1], d["signs"], radices, d["thetas"], d["base_mixers"])

    w.oracle = oracle
    if host_only:
        return w
    import hadamard_incoherence_transforms_b200 as hit

    x = torch.from_numpy(d["x"]).to(dev)
    s = torch.from_numpy(d["signs"]).to(dev)
    th = [torch.from_numpy(t).to(dev) for t in d["thetas"]]
    blocks = [torch.empty((n // b, b, b), dtype=torch.float32, device=dev) for b in radices]
    y = torch.empty_like(x)
    w.rotation = 1

    def step(i):
        for t, b in enumerate(radices):
            hit.harp_blocks(th[t], b, signs=s if t == 0 else None, out=blocks[t])
        hit.butterfly_apply(x, radices, blocks, out=y)

    w.step = step
    w.parity = lambda ref, r0, r1: {"rows": r1 - r0, "rel_l2": _rel_l2(_host64(y[r0:r1]), ref)}
    hx = x.cpu().pin_memory()
    hy = torch.empty_like(hx).pin_memory()

    def e2e_step(i):
        x.copy_(hx, non_blocking=True)
        step(i)
        hy.copy_(y, non_blocking=True)

    w.e2e_step = e2e_step
    return w


WORKLOADS = {
    "weight_rht_int4": weight_rht_int4,
    "activation_quant": activation_quant,
    "activation_rht": activation_rht,
    "two_sided_lowbit": two_sided_lowbit,
    "wht_adapter": wht_adapter,
    "two_sided_butterfly": two_sided_butterfly,
    "mixed_rht_int4": mixed_rht_int4,
    "harp_rotation": harp_rotation,
}


# ----------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ----------------------------------------------------------------------------
def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def time_oracle(w, budget_s: float, chunk: int) -> tuple[float, int, float]:
    """Run the oracle on consecutive row chunks (wrapping around the workload)
    until `budget_s` of CPU time has elapsed.  Returns (seconds, rows, rows/s)."""
    t0 = time.perf_counter()
    done = 0
    while (time.perf_counter() - t0) < budget_s:
        r0 = done % w.rows
        r1 = min(w.rows, r0 + chunk)
        w.oracle(r0, r1)
        done += r1 - r0
    dt = time.perf_counter() - t0
    return dt, done, done / dt


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload](None, 0, host_only=True, bits=args.bits)
    per_row = w.bytes / w.rows
    # size one step's sample so warmup + steps finish within about two minutes
    t0 = time.perf_counter()
    w.oracle(0, 1)
    t_row = max(time.perf_counter() - t0, 1e-4)
    sample = int(max(1, min(w.rows, 120.0 / max(1, args.steps + args.warmup) / t_row)))
    for i in range(args.warmup):
        r0 = (i * sample) % max(1, w.rows - sample + 1)
        w.oracle(r0, r0 + sample)
    times = []
    for i in range(args.steps):
        r0 = (i * sample) % max(1, w.rows - sample + 1)
        t = time.perf_counter()
        w.oracle(r0, r0 + sample)
        times.append(time.perf_counter() - t)
    sec = float(np.mean(times))
    value = per_row * sample / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.desc, "rows_per_step": sample, "n": w.n},
        "rows_per_s": sample / sec,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"{sample} rows of {w.rows} per step (numpy float64 dense Hadamard + fp32 quantizer)"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
def capture_steps(w, steps, first):
    """Capture `steps` consecutive steps (rotation sets first, first+1, ...) into
    one CUDA graph, so the timed region replays the kernels back to back with
    no host-side launch overhead between them."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for i in range(steps):
                w.step(first + i)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    return g


def time_region(g, stream):
    """Replay the K-step graph between two events on the launching stream.

    A spin kernel queued ahead of the start event keeps the GPU busy while the
    host submits the event and the graph, so the timed region starts when the
    graph's first kernel can start (host submission latency, ~25 us per replay,
    is not GPU time of the K steps)."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(200_000)  # ~0.1 ms at 1.9 GHz, before the start event
    start.record(stream)
    g.replay()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def run_gpu(args, world, rank, local):
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    import hadamard_incoherence_transforms_b200 as hit

    hit.load()  # fails loudly if the extension is missing
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    w = WORKLOADS[args.workload](dev, l2, bits=args.bits)

    for i in range(args.warmup):
        w.step(i)
    torch.cuda.synchronize()
    graph = capture_steps(w, args.steps, args.warmup)
    stream = torch.cuda.current_stream(dev)
    # The first launch of a captured graph also uploads it to the device;
    # replay it once untimed so the timed replay measures the kernels only.
    graph.replay()
    torch.cuda.synchronize()
    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms = time_region(graph, stream)
        barrier(dist)
        torch.cuda.synchronize()
    del graph
    total_ms = reduce_max(total_ms, dist, dev)
    ms_step = total_ms / args.steps
    value = world * w.bytes / (ms_step * 1e-3) / 1e9
    # The graph runs the step's kernels back to back, so for a one-kernel step
    # (the headline) the step time is that kernel's average launch duration.
    # A multi-kernel step's roofline block covers the whole step instead; its
    # per-kernel split is in the committed launch lists.
    kern_ms = ms_step
    achieved = w.bytes / (kern_ms * 1e-3) / 1e9

    # end-to-end through the public API with pinned host buffers
    e2e_steps = max(3, min(args.steps, 20))
    for i in range(2):
        w.e2e_step(i)
    torch.cuda.synchronize()
    barrier(dist)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(e2e_steps):
        w.e2e_step(i)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(a.elapsed_time(b) / e2e_steps, dist, dev)
    e2e_value = world * w.bytes / (e2e_ms * 1e-3) / 1e9

    peak, peak_kind = measured_peaks()
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.desc, "io": w.io, "rows": w.rows, "n": w.n,
                   "l2": f"rotating {w.rotation} input/output sets ({w.rotation * w.bytes / 1e6:.0f} MB) vs L2 {l2 / 1e6:.0f} MB",
                   "parallelism": f"replicas x{world}"},
        "rows_per_s": world * w.rows / (ms_step * 1e-3),
        "pct_of_peak_hbm": 100.0 * value / (world * peak),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": read_profile_traffic(w.kernel_key) if w.kernels_per_step == 1 else None,
                     "kernel": w.kernel_key if w.kernels_per_step == 1 else f"whole step ({w.kernels_per_step} kernels)"},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": w.h2d, "d2h_bytes_per_step": w.d2h},
        "gpu_launches": args.steps * w.kernels_per_step,
        "clocks": clk.summary(),
    }
    if hasattr(w, "extra"):
        line.update(w.extra())
    # bounded device waits that gave up during the run (0 = every output defined)
    line["wait_timeouts"] = hit.wait_timeouts()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, rows_done, rps = time_oracle(w, budget_s=args.cpu_budget, chunk=max(1, min(256, w.rows)))
        line["cpu_baseline"] = {"value": rps * w.bytes / w.rows / 1e9, "unit": "GB/s", "cores": cpu_threads(),
                                "kind": "oracle",
                                "sample": f"{rows_done} rows of the {w.rows}-row workload (wrapping) in {sec:.1f} s, scaled to GB/s"}
        # parity of the timed outputs on the first rows, against the oracle's
        k = min(8, w.rows)
        line["cpu_baseline"]["parity"] = w.parity(w.oracle(0, k), 0, k)
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def relaunch(n: int, argv=None) -> int:
    """Run this script under torch.distributed.run with n ranks on this node."""
    import socket
    import subprocess

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)]
    cmd += list(sys.argv[1:] if argv is None else argv)
    return subprocess.call(cmd)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["hit", "reference"], default="hit")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="weight_rht_int4")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bits", type=int, choices=[2, 3], default=3, help="code width of two_sided_lowbit")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_env()
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return relaunch(args.gpus, argv)
    if args.gpus != world:
        print(json.dumps({"error": f"--gpus {args.gpus} but WORLD_SIZE is {world}"}))
        return 2
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_gpu(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
