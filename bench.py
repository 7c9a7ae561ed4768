"""Benchmark of the Hadamard-rotation + block-quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extras] [--schedule fused|two_pass]

One JSON line on stdout (rank 0).  The headline workload is the grouped MoE
NVFP4 cast: BF16 [16384, 7168], 32 split sections, 16-point RHT on the
columnwise output, rowwise + columnwise E2M1 codes with E4M3 1x16 block
scales and per-section FP32 amax / global scale.  `value` is whole-job HBM
throughput in GB/s of algorithmic bytes (input read once + outputs written
once) with inputs resident on the device; `e2e` is the same metric through
the C ABI with pinned host buffers and the copies inside the timed region.
The other workloads of the path (dense NVFP4, DSA indexer FP8, QMoE K128 FP8
of BF16 and of SwiGLU) are reported under "workloads".

Timing: W untimed warm-up steps, then exactly K steps on the launching
stream between CUDA events; barrier + synchronize around the timed region;
the step time is the max over ranks.  Inputs larger than L2 run the K steps
back to back (no step finds its inputs in L2).  Smaller inputs get an L2
flush before every step, outside the events: a 256 MiB write, then a 256 MiB
read of another buffer, so that the step starts with none of its inputs and
no dirty line in L2 (with the write alone, up to 126 MB of the flush's own
dirty lines would be written back inside the timed step).  Under torchrun every rank quantizes its
own batch (independent problems, no collective on the data path: weak
scaling); torch.distributed only carries the barrier and the max of the times.

--impl reference times the CPU oracle (the reference implementation of the
pages' arithmetic, plain single-threaded C) on the host cores: for the grouped
workloads each step is the whole workload, its sections and directions spread
over all host cores; for the others each step is a bounded sample on one core.
Rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "RHT+block-quant HBM GB/s & % of peak, grouped NVFP4 16384x7168"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="grouped_moe",
                    choices=("grouped_moe", "grouped_moe_amax_given", "grouped_moe_row_rht", "grouped_moe_sr",
                             "grouped_moe_sf_interleaved", "dense_nvfp4", "dsa_indexer", "dsa_indexer_ue8m0",
                             "dsa_indexer_nvfp4", "qmoe_bf16", "qmoe_swiglu", "fp8_single"))
    ap.add_argument("--no-extras", action="store_true", help="time only the headline workload")
    ap.add_argument("--schedule", choices=("fused", "two_pass"), default="fused")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- ranks
class Ranks:
    """RANK / WORLD_SIZE from the environment; torch.distributed for N > 1."""

    def __init__(self):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend: str):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, value: float, device) -> float:
        if not self.pg:
            return value
        import torch
        import torch.distributed as dist
        t = torch.tensor([value], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            for r in csv.reader(io.StringIO(open(self.path).read())):
                if len(r) >= 9:
                    rows.append([c.strip() for c in r])
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = sorted(v for v in (num(r[1]) for r in rows) if v is not None)
        smax = max((v for v in (num(r[2]) for r in rows) if v is not None), default=None)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ---------------------------------------------------------------- peaks
def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


def kernel_source_sha() -> str:
    """Hash of the CUDA sources: ncu traffic figures are only valid for the
    kernels they were captured on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_quantization_group_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from profiles/traffic.txt ("workload sha bytes"),
    or None when missing or captured on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    sha = kernel_source_sha()
    try:
        for line in open(path):
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == workload and parts[1] == sha:
                return int(parts[2])
    except OSError:
        pass
    return None


# ------------------------------------------------------------- workloads
class Workload:
    """One configuration of the path: inputs, outputs, the timed call."""

    name = ""
    launches_per_step = 1

    def __init__(self, rank: int):
        self.rank = rank

    # host side ------------------------------------------------------
    def host_inputs(self) -> dict:          # name -> numpy array
        raise NotImplementedError

    def alg_bytes(self) -> int:             # input read once + outputs written once
        raise NotImplementedError

    def elements(self) -> int:
        raise NotImplementedError

    def config(self) -> dict:
        raise NotImplementedError

    # device side ----------------------------------------------------
    def setup(self, hq, torch, host: dict):
        self.hq, self.torch = hq, torch
        self.dev_in = {k: self._to_dev(torch, v) for k, v in host.items()}
        self.out = self.alloc_outputs(torch)

    @staticmethod
    def _to_dev(torch, a):
        t = torch.from_numpy(a)
        if t.dtype == torch.uint16:
            t = t.view(torch.bfloat16)
        return t.cuda()

    def alloc_outputs(self, torch) -> dict:
        raise NotImplementedError

    def call(self, inputs: dict, out: dict) -> None:
        raise NotImplementedError

    def step(self):
        self.call(self.dev_in, self.out)

    # end to end: pinned host buffers, copies inside the timed region
    def setup_e2e(self, host: dict):
        torch = self.torch
        self.h_in = {k: self._pinned(torch, v) for k, v in host.items()}
        self.h_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in self.out.items()}
        self.e2e_in = {k: torch.empty_like(v) for k, v in self.dev_in.items()}

    @staticmethod
    def _pinned(torch, a):
        t = torch.from_numpy(a)
        if t.dtype == torch.uint16:
            t = t.view(torch.bfloat16)
        return t.pin_memory()

    def e2e_step(self):
        for k, v in self.h_in.items():
            self.e2e_in[k].copy_(v, non_blocking=True)
        self.call(self.e2e_in, self.out)
        for k, v in self.out.items():
            self.h_out[k].copy_(v, non_blocking=True)

    def input_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.dev_in.values())

    def h2d_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.h_in.values())

    def d2h_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.h_out.values())

    # oracle sample --------------------------------------------------
    def oracle_sample(self, host: dict):
        """(callable, bytes, description): a bounded slice of the workload."""
        raise NotImplementedError


class GroupedNVFP4(Workload):
    name = "grouped_moe"

    def __init__(self, rank, M=16384, K=7168, sections=32, schedule="fused", seed_key="grouped_moe"):
        super().__init__(rank)
        import synthetic as S
        self.M, self.K = M, K
        self.seed = S.SEEDS[seed_key] + 97 * rank
        self.splits = S.moe_splits(self.seed, total_rows=M, sections=sections) if sections > 1 else [M]
        self.mask = S.sign_mask16(self.seed)
        self.schedule = schedule
        self.launches_per_step = 1 if schedule == "fused" else 2

    def host_inputs(self):
        import synthetic as S
        return {"x": S.normal_bf16(self.seed, (self.M, self.K))}

    def elements(self):
        return self.M * self.K

    def alg_bytes(self):
        # BF16 in (2 B) + row codes (0.5) + row sf (1/16) + col codes (0.5) + col sf (1/16)
        # + per section amax/sdec x 2 directions
        return self.elements() * 2 + 2 * (self.elements() // 2 + self.elements() // 16) + 16 * len(self.splits)

    def config(self):
        return {"workload": f"grouped MoE NVFP4 RHT16 cast, BF16 [{self.M},{self.K}], {len(self.splits)} sections",
                "M": self.M, "K": self.K, "sections": len(self.splits), "split_rows": self.splits,
                "sign_mask": self.mask, "directions": "rowwise+columnwise", "schedule": self.schedule}

    def alloc_outputs(self, torch):
        self.ws = self.hq.new_workspace(len(self.splits))
        return self.hq.group_outputs(self.M, self.K, len(self.splits))

    def flags(self):
        hq = self.hq
        return hq.HQ_ROWWISE | hq.HQ_COLWISE | (0 if self.schedule == "fused" else hq.HQ_TWO_PASS)

    sr_seed = None          # stochastic rounding seed of the host-buffer call (None: nearest)
    host_pipeline = True    # end to end through hq_group_rht_quant_host

    def call(self, inputs, out):
        hq = self.hq
        hq.hq_group_rht_quant(inputs["x"], self.M, self.K, self.splits, len(self.splits), self.mask, self.flags(),
                              out["row_codes"], out["row_sf"], out["col_codes"], out["col_sf"],
                              out["amax_row"], out["amax_col"], out["sdec_row"], out["sdec_col"], self.ws)

    # end to end: the host-buffer entry, which overlaps the copies in, the
    # casts and the copies out by groups of whole sections
    def setup_e2e(self, host):
        if not self.host_pipeline:
            return super().setup_e2e(host)
        torch, hq = self.torch, self.hq
        self.h_in = {"x": self._pinned(torch, host["x"])}
        self.h_out = hq.host_outputs(self.M, self.K, len(self.splits), self.flags())
        self.staging = hq.HostStaging(self.M, self.K, len(self.splits))

    def e2e_step(self):
        if not self.host_pipeline:
            return super().e2e_step()
        self.hq.group_rht_quant_host(self.h_in["x"], self.splits, self.mask, self.flags(), staging=self.staging,
                                     out=self.h_out, seed=self.sr_seed)

    def oracle_sample(self, host, rows=512):
        import oracle
        # rows 0..rows-1 of the workload's input, quantized as one section
        x = host["x"][:rows]
        return (lambda: oracle.group_rht_quant(x, [rows], self.mask, oracle.ROWWISE | oracle.COLWISE),
                rows * self.K * 2 + 2 * (rows * self.K // 2 + rows * self.K // 16),
                f"one {rows}-row section of the BF16 [{self.M},{self.K}] input (rows 0..{rows - 1})")


    def oracle_full(self, host, cores):
        """(callable, bytes, description): the whole workload on `cores` host
        threads.  Each task is one direction of one non-empty section (the
        oracle's unit: a section's amax needs all its rows); tasks run longest
        first, and ctypes releases the GIL while the C oracle runs."""
        import oracle
        from concurrent.futures import ThreadPoolExecutor
        x = host["x"]
        tasks, r0 = [], 0
        for Ms in self.splits:
            if Ms:
                for d in (oracle.ROWWISE, oracle.COLWISE):
                    tasks.append((Ms, r0, d))
            r0 += Ms
        tasks.sort(reverse=True)

        def one(t):
            Ms, r, d = t
            oracle.group_rht_quant(x[r:r + Ms], [Ms], self.mask, d)

        def run():
            with ThreadPoolExecutor(max_workers=cores) as ex:
                list(ex.map(one, tasks))
        return (run, self.alg_bytes(),
                f"the whole workload (all {len(self.splits)} sections), {len(tasks)} section-direction tasks "
                f"on {cores} threads")


class GroupedInterleavedSF(GroupedNVFP4):
    """The grouped cast with its block scales in the interleaved 128 x 4 tiles
    block-scaled tcgen05 MMAs read (HQ_SF_SWIZZLED)."""
    name = "grouped_moe_sf_interleaved"
    host_pipeline = False

    def config(self):
        c = super().config()
        c["workload"] += ", block scales in interleaved 128x4 tiles"
        return c

    def flags(self):
        return super().flags() | self.hq.HQ_SF_SWIZZLED

    def oracle_sample(self, host, rows=512):
        import oracle
        x = host["x"][:rows]
        flags = oracle.ROWWISE | oracle.COLWISE | oracle.SF_SWIZZLED
        return (lambda: oracle.group_rht_quant(x, [rows], self.mask, flags),
                rows * self.K * 2 + 2 * (rows * self.K // 2 + rows * self.K // 16),
                f"one {rows}-row section of the BF16 [{self.M},{self.K}] input, interleaved block scales")


class GroupedAmaxGiven(GroupedNVFP4):
    """The same workload with the section amax values supplied by the caller
    (HQ_AMAX_GIVEN): one pass over x.  The amax values come from one ordinary
    call before the timed steps."""
    name = "grouped_moe_amax_given"
    host_pipeline = False   # (its amax inputs stay on the device)

    def setup(self, hq, torch, host):
        super().setup(hq, torch, host)
        GroupedNVFP4.call(self, self.dev_in, self.out)   # fills amax_row / amax_col
        torch.cuda.synchronize()

    def config(self):
        c = super().config()
        c["workload"] += ", section amax given (single pass)"
        c["schedule"] = "amax given"
        return c

    def call(self, inputs, out):
        hq = self.hq
        hq.hq_group_rht_quant(inputs["x"], self.M, self.K, self.splits, len(self.splits), self.mask,
                              hq.HQ_ROWWISE | hq.HQ_COLWISE | hq.HQ_AMAX_GIVEN,
                              out["row_codes"], out["row_sf"], out["col_codes"], out["col_sf"],
                              out["amax_row"], out["amax_col"], out["sdec_row"], out["sdec_col"], self.ws)

    def oracle_sample(self, host, rows=512):
        import oracle
        x = host["x"][:rows]
        r = oracle.group_rht_quant(x, [rows], self.mask, oracle.ROWWISE | oracle.COLWISE)
        flags = oracle.ROWWISE | oracle.COLWISE | oracle.AMAX_GIVEN
        return (lambda: oracle.group_rht_quant(x, [rows], self.mask, flags, amax_row=r["amax_row"],
                                               amax_col=r["amax_col"]),
                rows * self.K * 2 + 2 * (rows * self.K // 2 + rows * self.K // 16),
                f"one {rows}-row section of the BF16 [{self.M},{self.K}] input, amax given")


class GroupedRowRHT(GroupedNVFP4):
    """The same workload with the rowwise output rotated too (HQ_ROW_RHT)."""
    name = "grouped_moe_row_rht"

    def config(self):
        c = super().config()
        c["workload"] += ", rowwise output rotated too"
        c["directions"] = "rowwise (RHT16 along K) + columnwise"
        return c

    def flags(self):
        return super().flags() | self.hq.HQ_ROW_RHT

    def oracle_sample(self, host, rows=512):
        import oracle
        x = host["x"][:rows]
        flags = oracle.ROWWISE | oracle.COLWISE | oracle.ROW_RHT
        return (lambda: oracle.group_rht_quant(x, [rows], self.mask, flags),
                rows * self.K * 2 + 2 * (rows * self.K // 2 + rows * self.K // 16),
                f"one {rows}-row section of the BF16 [{self.M},{self.K}] input, rows rotated too")


class GroupedSR(GroupedNVFP4):
    """The same workload with stochastic rounding of both directions' codes
    (hq_group_rht_quant_sr, Philox4x32-10 random bytes)."""
    name = "grouped_moe_sr"

    def config(self):
        c = super().config()
        c["workload"] += ", stochastic rounding (rowwise and columnwise codes)"
        return c

    sr_seed = 1234

    def flags(self):
        hq = self.hq
        return hq.HQ_ROWWISE | hq.HQ_COLWISE | hq.HQ_ROW_SR | hq.HQ_COL_SR

    def call(self, inputs, out):
        hq = self.hq
        hq.hq_group_rht_quant_sr(inputs["x"], self.M, self.K, self.splits, len(self.splits), self.mask,
                                 self.flags(), self.sr_seed, 0,
                                 out["row_codes"], out["row_sf"], out["col_codes"], out["col_sf"],
                                 out["amax_row"], out["amax_col"], out["sdec_row"], out["sdec_col"], self.ws)

    def oracle_sample(self, host, rows=512):
        import oracle
        x = host["x"][:rows]
        flags = oracle.ROWWISE | oracle.COLWISE | oracle.ROW_SR | oracle.COL_SR
        return (lambda: oracle.group_rht_quant(x, [rows], self.mask, flags, seed=1234, offset=0),
                rows * self.K * 2 + 2 * (rows * self.K // 2 + rows * self.K // 16),
                f"one {rows}-row section of the BF16 [{self.M},{self.K}] input, stochastic rounding")


class DenseNVFP4(GroupedNVFP4):
    name = "dense_nvfp4"

    def __init__(self, rank, schedule="fused"):
        super().__init__(rank, M=8192, K=4096, sections=1, schedule=schedule, seed_key="dense_nvfp4")
        # one section of 2048 tiles (more than a wave of the grid): the library
        # takes two launches, the streaming amax kernel and the casts
        self.launches_per_step = 2

    def host_inputs(self):
        import synthetic as S
        return {"x": S.with_outliers_bf16(S.normal_bf16(self.seed, (self.M, self.K)), self.seed + 1, 0.001, 50.0)}

    def config(self):
        c = super().config()
        c["workload"] = "dense NVFP4 RHT16 cast, BF16 [8192,4096], 0.1% x50 outliers"
        c["schedule"] = "two launches (one section: the library's choice)"
        return c


class DSAIndexer(Workload):
    name = "dsa_indexer"

    def __init__(self, rank, T=4096, H=64):
        super().__init__(rank)
        import synthetic as S
        self.T, self.H = T, H
        self.seed = S.SEEDS["dsa_indexer"] + 97 * rank

    def host_inputs(self):
        import synthetic as S
        return {"pe": S.normal_bf16(self.seed, (self.T, self.H, 64)),
                "nope": S.normal_bf16(self.seed + 100, (self.T, self.H, 64))}

    def elements(self):
        return self.T * self.H * 128

    def alg_bytes(self):
        return self.elements() * 2 + self.elements() + self.T * self.H * 4

    def config(self):
        return {"workload": f"DSA indexer prep: cat q_pe|q_nope BF16 [{self.T},{self.H},64]x2 -> H128 -> FP8 1x128, "
                            f"scales [{self.H},{self.T}]"}

    def alloc_outputs(self, torch):
        return {"codes": torch.empty((self.T, self.H * 128), dtype=torch.uint8, device="cuda"),
                "scales": torch.empty((self.H, self.T), dtype=torch.float32, device="cuda")}

    def call(self, inputs, out):
        self.hq.hq_cat_rotate_fp8(inputs["pe"], self.H * 64, 64, inputs["nope"], self.H * 64, 64, self.T, self.H,
                                  128, out["codes"], out["scales"], self.hq.HQ_SCALE_TRANSPOSED, self.T)

    def oracle_sample(self, host, tokens=256):
        import oracle
        pe, nope = host["pe"][:tokens], host["nope"][:tokens]
        return (lambda: oracle.cat_rotate_fp8(pe, nope, tokens, self.H, 128, scale_layout=oracle.TRANSPOSED,
                                              scale_ld=tokens),
                tokens * self.H * (128 * 3 + 4), f"tokens 0..{tokens - 1} of the [{self.T},{self.H}] indexer input")


class DSAIndexerNVFP4(DSAIndexer):
    """The same indexer input, NVFP4 per rotated 128-vector (codes, E4M3 block
    scales, per-vector decode scales transposed)."""
    name = "dsa_indexer_nvfp4"

    def alg_bytes(self):
        # BF16 in (2) + codes (0.5) + block scales (1/16) per element + a float per vector
        return self.elements() * 2 + self.elements() // 2 + self.elements() // 16 + self.T * self.H * 4

    def config(self):
        return {"workload": f"DSA indexer prep, FP4: cat q_pe|q_nope BF16 [{self.T},{self.H},64]x2 -> H128 -> NVFP4 "
                            f"per 128-vector, vector scales [{self.H},{self.T}]"}

    def alloc_outputs(self, torch):
        return {"codes": torch.empty((self.T, self.H * 64), dtype=torch.uint8, device="cuda"),
                "block_sf": torch.empty((self.T, self.H * 8), dtype=torch.uint8, device="cuda"),
                "sdec": torch.empty((self.H, self.T), dtype=torch.float32, device="cuda")}

    def call(self, inputs, out):
        self.hq.hq_cat_rotate_nvfp4(inputs["pe"], self.H * 64, 64, inputs["nope"], self.H * 64, 64, self.T, self.H,
                                    128, out["codes"], out["block_sf"], out["sdec"], self.hq.HQ_SCALE_TRANSPOSED,
                                    self.T)

    def oracle_sample(self, host, tokens=256):
        import oracle
        pe, nope = host["pe"][:tokens], host["nope"][:tokens]
        return (lambda: oracle.cat_rotate_nvfp4(pe, nope, tokens, self.H, 128, scale_layout=oracle.TRANSPOSED,
                                                scale_ld=tokens),
                tokens * self.H * 128 * 2 + tokens * self.H * (64 + 8 + 4),
                f"tokens 0..{tokens - 1} of the [{self.T},{self.H}] indexer input")


class DSAIndexerUE8M0(DSAIndexer):
    """The indexer prep with UE8M0 (power-of-two) FP8 scales."""
    name = "dsa_indexer_ue8m0"

    def config(self):
        c = super().config()
        c["workload"] += ", UE8M0 scales"
        return c

    def call(self, inputs, out):
        hq = self.hq
        hq.hq_cat_rotate_fp8(inputs["pe"], self.H * 64, 64, inputs["nope"], self.H * 64, 64, self.T, self.H,
                             128, out["codes"], out["scales"], hq.HQ_SCALE_TRANSPOSED | hq.HQ_FP8_UE8M0, self.T)

    def oracle_sample(self, host, tokens=256):
        import oracle
        pe, nope = host["pe"][:tokens], host["nope"][:tokens]
        return (lambda: oracle.cat_rotate_fp8(pe, nope, tokens, self.H, 128,
                                              scale_layout=oracle.TRANSPOSED | oracle.UE8M0, scale_ld=tokens),
                tokens * self.H * (128 * 3 + 4), f"tokens 0..{tokens - 1} of the [{self.T},{self.H}] indexer input")


class FP8Single(DSAIndexer):
    name = "fp8_single"

    def __init__(self, rank):
        Workload.__init__(self, rank)
        import synthetic as S
        self.T, self.H = 512, 1
        self.seed = S.SEEDS["fp8_single"] + 97 * rank

    def host_inputs(self):
        import synthetic as S
        return {"x": S.normal_bf16(self.seed, (512, 1, 128))}

    def config(self):
        return {"workload": "BF16 [512,128] -> H128 -> FP8 1x128 (launch-bound, correctness case)"}

    def alloc_outputs(self, torch):
        return {"codes": torch.empty((512, 128), dtype=torch.uint8, device="cuda"),
                "scales": torch.empty((512, 1), dtype=torch.float32, device="cuda")}

    def call(self, inputs, out):
        self.hq.hq_cat_rotate_fp8(inputs["x"], 128, 128, None, 0, 0, 512, 1, 128, out["codes"], out["scales"],
                                  self.hq.HQ_SCALE_ROWMAJOR, 1)

    def oracle_sample(self, host):
        import oracle
        x = host["x"]
        return (lambda: oracle.cat_rotate_fp8(x, None, 512, 1, 128), 512 * (128 * 3 + 4), "the whole [512,128] input")


class QMoE(Workload):
    def __init__(self, rank, swiglu: bool, M=32768, K=4096):
        super().__init__(rank)
        import synthetic as S
        self.swiglu = swiglu
        self.name = "qmoe_swiglu" if swiglu else "qmoe_bf16"
        self.M = M
        self.K_in = K                       # 4096 input columns (BF16) or gate|up 2 x 2048 (FP32)
        self.K_out = K // 2 if swiglu else K
        self.seed = S.SEEDS["qmoe"] + (100 if swiglu else 0) + 97 * rank

    def host_inputs(self):
        import synthetic as S
        if self.swiglu:
            return {"x": S.normal_f32(self.seed, (self.M, self.K_in), std=2.0 ** 0.5)}
        return {"x": S.normal_bf16(self.seed, (self.M, self.K_in))}

    def elements(self):
        return self.M * self.K_out

    def alg_bytes(self):
        in_bytes = self.M * self.K_in * (4 if self.swiglu else 2)
        return in_bytes + self.M * self.K_out + self.M * (self.K_out // 128) * 4

    def config(self):
        what = (f"FP32 gate|up [{self.M},2x{self.K_out}] -> SiLU(gate)*up -> K128 FP8" if self.swiglu
                else f"BF16 [{self.M},{self.K_in}] -> K128 FP8")
        return {"workload": f"QMoE dynamic FP8 activations: {what}"}

    def alloc_outputs(self, torch):
        return {"codes": torch.empty((self.M, self.K_out), dtype=torch.uint8, device="cuda"),
                "scales": torch.empty((self.M, self.K_out // 128), dtype=torch.float32, device="cuda")}

    def call(self, inputs, out):
        hq = self.hq
        mode = hq.HQ_ACT_SWIGLU_F32 if self.swiglu else hq.HQ_ACT_NONE_BF16
        hq.hq_swiglu_fp8_k128(mode, inputs["x"], self.M, self.K_out, out["codes"], out["scales"])

    def oracle_sample(self, host, rows=2048):
        import oracle
        x = host["x"][:rows]
        mode = oracle.SWIGLU_F32 if self.swiglu else oracle.NONE_BF16
        nbytes = rows * self.K_in * (4 if self.swiglu else 2) + rows * self.K_out + rows * (self.K_out // 128) * 4
        return (lambda: oracle.swiglu_fp8_k128(mode, x, rows, self.K_out), nbytes, f"rows 0..{rows - 1}")


def make_workload(name: str, rank: int, schedule: str = "fused") -> Workload:
    return {"grouped_moe": lambda: GroupedNVFP4(rank, schedule=schedule),
            "grouped_moe_amax_given": lambda: GroupedAmaxGiven(rank),
            "grouped_moe_sf_interleaved": lambda: GroupedInterleavedSF(rank, schedule=schedule),
            "dsa_indexer_ue8m0": lambda: DSAIndexerUE8M0(rank),
            "grouped_moe_row_rht": lambda: GroupedRowRHT(rank, schedule=schedule),
            "grouped_moe_sr": lambda: GroupedSR(rank, schedule=schedule),
            "dense_nvfp4": lambda: DenseNVFP4(rank, schedule=schedule),
            "dsa_indexer": lambda: DSAIndexer(rank),
            "dsa_indexer_nvfp4": lambda: DSAIndexerNVFP4(rank),
            "fp8_single": lambda: FP8Single(rank),
            "qmoe_bf16": lambda: QMoE(rank, swiglu=False),
            "qmoe_swiglu": lambda: QMoE(rank, swiglu=True)}[name]()


def sample_inputs(wl: Workload) -> dict:
    """The leading slice of the workload's inputs that its oracle sample uses.
    The generator is counter-based, so a prefix of the stream is exactly the
    first rows of the full tensor."""
    import synthetic as S
    if isinstance(wl, GroupedNVFP4):
        rows = 512
        x = S.normal_bf16(wl.seed, (rows, wl.K))
        if isinstance(wl, DenseNVFP4):
            x = S.with_outliers_bf16(x, wl.seed + 1, 0.001, 50.0)
        return {"x": x}
    if isinstance(wl, FP8Single):
        return wl.host_inputs()
    if isinstance(wl, DSAIndexer):
        n = 256 * wl.H * 64
        return {"pe": S.normal_bf16(wl.seed, (n,)).reshape(256, wl.H, 64),
                "nope": S.normal_bf16(wl.seed + 100, (n,)).reshape(256, wl.H, 64)}
    if isinstance(wl, QMoE):
        rows = 2048
        if wl.swiglu:
            return {"x": S.normal_f32(wl.seed, (rows * wl.K_in,), std=2.0 ** 0.5).reshape(rows, wl.K_in)}
        return {"x": S.normal_bf16(wl.seed, (rows * wl.K_in,)).reshape(rows, wl.K_in)}
    raise ValueError(wl.name)


# ----------------------------------------------------------------- timing
def l2_bytes(torch) -> int:
    return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)


class L2Flush:
    """Before a step: write a buffer larger than L2, then read another one, so
    that L2 holds neither the step's inputs nor dirty lines to write back."""

    def __init__(self, torch):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def time_device(torch, wl: Workload, steps: int, warmup: int, ranks: Ranks, flush, force_flush=False):
    """Per-step milliseconds and how L2 was handled.  Inputs larger than L2:
    the steps run back to back (a step finds none of its inputs in L2; its own
    outputs' write-back is part of its traffic).  Smaller inputs: a 256 MiB
    write and a 256 MiB read flush L2 before every step, outside the timed
    events."""
    stream = torch.cuda.current_stream()
    l2 = l2_bytes(torch)
    if wl.input_bytes() > l2 and not force_flush:
        for _ in range(warmup):
            wl.step()
        torch.cuda.synchronize()
        ranks.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(400000)          # GPU-side wait (no memory traffic) while the host enqueues the steps
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            wl.step()
        b.record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
        torch.cuda.synchronize()
        note = (f"inputs ({wl.input_bytes() / 1e6:.0f} MB) larger than L2 ({l2 / 1e6:.0f} MB): steps back to back, "
                "no flush")
        return [a.elapsed_time(b) / steps] * steps, note
    for _ in range(warmup):
        flush()
        wl.step()
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush()                            # L2 flush, outside the timed events
        a.record(stream)
        wl.step()
        b.record(stream)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs], (f"flushed before every step ({L2_FLUSH_BYTES >> 20} MiB write, then "
                                                 f"{L2_FLUSH_BYTES >> 20} MiB read of another buffer)")


def time_e2e(torch, wl: Workload, steps: int, warmup: int, ranks: Ranks) -> list:
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        wl.e2e_step()
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        wl.e2e_step()
        b.record(stream)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def full_oracle_ok(wl) -> bool:
    """The grouped workloads (nearest rounding, computed amax) time the oracle on the whole workload."""
    return type(wl) in (GroupedNVFP4, DenseNVFP4)


def time_oracle(fn, min_seconds: float) -> tuple:
    """Run fn until min_seconds have passed (at least once); mean seconds per call."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            return el / n, n


def gbs(nbytes: float, ms: float) -> float:
    return nbytes / (ms * 1e-3) / 1e9


def mean(xs):
    return sum(xs) / len(xs)


# -------------------------------------------------------------- the arms
def run_reference(args, ranks: Ranks) -> None:
    """The oracle on the host cores: each step one bounded sample."""
    if ranks.rank != 0:
        return
    import oracle
    oracle.build()
    wl = make_workload(args.workload, 0, args.schedule)
    cores = 1
    if full_oracle_ok(wl):
        cores = host_cores()
        fn, nbytes, desc = wl.oracle_full(wl.host_inputs(), cores)
    else:
        fn, nbytes, desc = wl.oracle_sample(sample_inputs(wl))
    for _ in range(args.warmup):
        fn()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    ms = mean(times) * 1e3
    v = gbs(nbytes, ms)
    line = {"impl": "reference", "metric": METRIC if wl.name == "grouped_moe" else f"{wl.name} GB/s",
            "value": round(v, 4), "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": dict(wl.config(), l2="host cores (the oracle)",
                           parallelism=f"{args.gpus} independent batch(es), rank 0 times the oracle",
                           alg_bytes_per_step_per_gpu=wl.alg_bytes(), elements_per_step_per_gpu=wl.elements()),
            "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{desc}; {nbytes} algorithmic bytes per step"},
            "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure(torch, hq, name, args, ranks, flush, with_e2e=False):
    wl = make_workload(name, ranks.rank, args.schedule)
    host = wl.host_inputs()
    wl.setup(hq, torch, host)
    ms, l2_note = time_device(torch, wl, args.steps, args.warmup, ranks, flush)
    step_ms = ranks.max(mean(ms), "cuda")
    res = {"wl": wl, "ms": step_ms, "ms_min": min(ms), "ms_all": ms, "l2": l2_note}
    if with_e2e and wl.input_bytes() > l2_bytes(torch):
        # the same steps with L2 flushed before each, for comparison
        msf, _ = time_device(torch, wl, args.steps, args.warmup, ranks, flush, force_flush=True)
        res["ms_flushed"] = ranks.max(mean(msf), "cuda")
    if with_e2e:
        wl.setup_e2e(host)
        e = time_e2e(torch, wl, args.steps, args.warmup, ranks)
        res["e2e_ms"] = ranks.max(mean(e), "cuda")
    res["host"] = host
    return res


def cpu_baseline(wl, host) -> dict:
    """The oracle timed on the host: on all cores over the whole workload (the
    grouped workloads), and on one core over a bounded sample."""
    import oracle
    oracle.build()
    fn, nbytes, desc = wl.oracle_sample(sample_inputs(wl))
    sec, n = time_oracle(fn, 8.0)
    one = {"value": round(nbytes / sec / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{desc}, {nbytes} algorithmic bytes, {n} runs, single-threaded C"}
    if not full_oracle_ok(wl):
        return one
    cores = host_cores()
    fn, nbytes, desc = wl.oracle_full(host, cores)
    sec, n = time_oracle(fn, 10.0)
    return {"value": round(nbytes / sec / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{desc}, {nbytes} algorithmic bytes, {n} runs", "single_core": one}


def run_ours(args, ranks: Ranks) -> None:
    import torch

    from nvfp4_quantization_group_b200 import _build
    _build.build()
    import nvfp4_quantization_group_b200 as hq
    hq.lib()  # fails loudly when the CUDA library is missing
    torch.cuda.set_device(ranks.local)
    ranks.init("nccl")
    peaks = measured_peaks()
    flush = L2Flush(torch)
    gpu_index = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        gpu_index = int(vis.split(",")[gpu_index])

    with ClockSampler(gpu_index) as clk:
        main = measure(torch, hq, args.workload, args, ranks, flush, with_e2e=not args.no_e2e)
    clocks = clk.summary()
    wl = main["wl"]
    world = ranks.world
    step_ms = main["ms"]
    value = gbs(wl.alg_bytes() * world, step_ms)
    per_launch_ms = step_ms / wl.launches_per_step
    achieved = gbs(wl.alg_bytes() / wl.launches_per_step, per_launch_ms)
    traffic = recorded_traffic(wl.name) if wl.launches_per_step == 1 else None
    line = {
        "metric": METRIC if wl.name == "grouped_moe" else f"{wl.name} GB/s",
        "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": dict(wl.config(), l2=main["l2"],
                       parallelism=f"{world} independent batch(es), one per GPU, no collective",
                       alg_bytes_per_step_per_gpu=wl.alg_bytes(), elements_per_step_per_gpu=wl.elements()),
        "elements_per_s": round(wl.elements() * world / (step_ms * 1e-3), 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "peak_source": f"{peaks['source']} (copy bandwidth)",
                     "kernel": "nvfp4_group_kernel" if isinstance(wl, GroupedNVFP4) else wl.name},
        "clocks": clocks,
        "gpu_launches": args.steps * wl.launches_per_step,
    }
    if "ms_flushed" in main:
        line["l2_flushed"] = {"ms_per_step": round(main["ms_flushed"], 5),
                              "value": round(gbs(wl.alg_bytes() * world, main["ms_flushed"]), 2),
                              "note": "the same steps with the L2 flush before each (outside the events)"}
    if "e2e_ms" in main:
        line["e2e"] = {"value": round(gbs(wl.alg_bytes() * world, main["e2e_ms"]), 3), "unit": UNIT,
                       "h2d_bytes_per_step": wl.h2d_bytes(), "d2h_bytes_per_step": wl.d2h_bytes(),
                       "ms_per_step": round(main["e2e_ms"], 4)}

    if ranks.rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, main["host"])

    # the other workloads of the path (device-resident, same timing rules)
    if not args.no_extras:
        host_main = main.pop("host")
        del main, host_main
        torch.cuda.empty_cache()
        extras = {}
        for name in ("grouped_moe_amax_given", "grouped_moe_row_rht", "grouped_moe_sr", "grouped_moe_sf_interleaved",
                     "dense_nvfp4", "dsa_indexer", "dsa_indexer_ue8m0", "dsa_indexer_nvfp4", "qmoe_bf16",
                     "qmoe_swiglu", "fp8_single"):
            if name == args.workload:
                continue
            r = measure(torch, hq, name, args, ranks, flush)
            w = r["wl"]
            extras[name] = {"config": w.config()["workload"], "l2": r["l2"],
                            "GB/s": round(gbs(w.alg_bytes() * world, r["ms"]), 2),
                            "ms_per_step": round(r["ms"], 5),
                            "frac_of_hbm": round(gbs(w.alg_bytes(), r["ms"]) / peaks["hbm_gbs"], 4),
                            "elements_per_s": round(w.elements() * world / (r["ms"] * 1e-3), 1),
                            "alg_bytes": w.alg_bytes(), "gpu_launches": args.steps * w.launches_per_step}
            line["gpu_launches"] += args.steps * w.launches_per_step
            del r, w
            torch.cuda.empty_cache()
        line["workloads"] = extras

    if ranks.rank == 0:
        print(json.dumps(line), flush=True)
    ranks.barrier()
    ranks.close()


def main(argv=None) -> int:
    args = parse_args(argv)
    ranks = Ranks()
    if args.impl == "reference":
        run_reference(args, ranks)
        return 0
    run_ours(args, ranks)
    return 0


if __name__ == "__main__":
    sys.exit(main())
