"""Benchmark: CKKS key-switched rotations/s on the rotation-batch workload.

Workload (one "step"): 64 ciphertexts at N = 2^16, L = 24 (one 60-bit + 23
40-bit primes), K = 8 special 60-bit primes, dnum = 3, each rotated by one of
16 seeded distinct steps in [1, 32767] with an evaluation key per step.  Each
rotation runs the whole key-switching path: automorphism, inverse NTT, ModUp
(base conversion + NTT), key inner product, ModDown (inverse NTT, centred
conversion, NTT, combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun every rank rotates its own 64 ciphertexts with its own copy of
the keys (independent work, no collective on the data path: weak scaling);
rank 0 prints one JSON line.  --impl reference times the CPU oracle on the
host cores on a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import seeded_inputs as S  # noqa: E402

LOG_N, L, K, DNUM = 16, 24, 8, 3
N_CTS, N_KEYS = 64, 16
LEVEL = 24
METRIC = "CKKS key-switched rotations/s (N=2^16,L=24,dnum=3); % of HBM roofline"
WORKLOAD = {"workload": "rotation batch: 64 fresh ciphertexts, 16 seeded rotation keys",
            "N": 1 << LOG_N, "L": L, "K": K, "dnum": DNUM, "level": LEVEL, "n_ciphertexts": N_CTS,
            "n_keys": N_KEYS, "l2": "inputs larger than L2 (1.6 GB of ciphertexts, 1.6 GB of keys per step)"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="default run: the rotation-batch line only, without the other workloads' entries")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--seeded-a", action="store_true",
                    help="keys with seeded a-halves (he_keygen_seeded_ex, HE_KEYGEN_SEEDED_A): only b stored, a "
                         "regenerated inside the key-switching kernels (rotation, hoisted, rotsum)")
    ap.add_argument("--case", default="rotation",
                    choices=["rotation", "ntt", "rot_small", "ps15_small", "ffn128", "ffn2048", "ps15", "tiny",
                             "hoisted", "rotsum", "attention"],
                    help="rotation: the headline workload (default). ffn128 / ffn2048 / ps15 / tiny: the other "
                         "workloads, one JSON line each. ntt / rot_small / ps15_small: kernel cases for profiler "
                         "captures (NTT of 512 limbs, 8 rotations with 2 keys, or the degree-15 evaluation of 8 "
                         "ciphertexts)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------------ inputs

def workload_inputs(master, primes_q, n_cts):
    steps = S.rotation_steps(master, N_KEYS, 1, (1 << (LOG_N - 1)) - 1)
    assign = S.step_assignment(master, n_cts, N_KEYS)
    return steps, [steps[u] for u in assign]


class ClockSampler:
    """SM clocks and clock-event reasons of this rank's GPU during the timed
    region, sampled every 20 ms through NVML (query only; nothing is set),
    or every 200 ms through nvidia-smi when NVML is unavailable.  The GPU is
    found by its PCI bus id, so the sample follows CUDA's device numbering
    whatever CUDA_VISIBLE_DEVICES holds."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.samples = []  # (sm MHz, max MHz, reasons bitmask) from NVML
        self.nvml = None
        self.stop_flag = threading.Event()

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.gpu)
        try:
            bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.nvml = (nv, h)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _poll(self):
        nv, h = self.nvml
        while not self.stop_flag.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                pass
            self.stop_flag.wait(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml:
            self.stop_flag.set()
            self.t.join(timeout=2)
            nv = self.nvml[0]
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            sm = [x[0] for x in self.samples]
            reasons = sorted({nm for x in self.samples for nm, b in bits.items() if x[2] & b})
            return {"sm_mhz": float(np.median(sm)) if sm else None,
                    "sm_max_mhz": float(self.samples[-1][1]) if self.samples else None,
                    "reasons": reasons, "samples": len(sm), "source": "nvml, 20 ms"}
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(self.NAMES, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 200 ms"}


# ------------------------------------------------------------ cpu baseline

def max_over_ranks(values, world, device):
    """Element-wise maximum of a list of floats over all ranks (the ranks'
    device times: the job's time is its slowest rank's)."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def rank_seed(master, rank):
    """Seed of a rank's own ciphertexts (every rank rotates different inputs)."""
    return master + 7919 * rank


class OracleRotations:
    """The oracle, as it stands, rotating full-size ciphertexts of the
    rotation-batch workload (uniform-residue ciphertexts at level 24, the
    workload's seeded steps and keys).  Keys are generated on first use,
    outside every timing."""

    def __init__(self):
        from oracle import ckks as C

        self.C = C
        master = S.master_seed(1)
        self.master = master
        self.P = C.Params(LOG_N, L, K, DNUM)
        _, self.ct_steps = workload_inputs(master, self.P.q, N_CTS)
        self.s = S.secret(master, self.P.N)
        self.uni = S.uniform_residues(master, "ct_residues", self.P.q, self.P.N, lead=(4, 2))
        self.keys = {}

    def key(self, st):
        if st not in self.keys:
            a, e = S.key_draws(self.master, self.P.galois_elt(st), self.P.mods, self.P.N, self.P.dnum)
            self.keys[st] = self.C.rotation_key(self.s, st, a, e, self.P)
        return self.keys[st]

    def rotate(self, i):
        """Rotation i of the batch (ciphertext i mod 64 with its step); returns seconds."""
        st = self.ct_steps[i % N_CTS]
        key = self.key(st)
        ct = self.C.make_ct(self.uni[i % 4], LEVEL, 2.0 ** 40)
        t0 = time.perf_counter()
        self.C.rotate(ct, st, key, self.P)
        return time.perf_counter() - t0


def cpu_baseline(seconds):
    """The oracle rotating full-size ciphertexts of this workload on the host
    cores until about `seconds` of rotation work has run (at least 2)."""
    o = OracleRotations()
    done, t_rot = 0, 0.0
    while (t_rot < seconds and done < 64) or done < 2:
        t_rot += o.rotate(done)
        done += 1
    return {"value": done / t_rot, "unit": "rotations/s", "cores": o.C.n_threads(), "kind": "oracle",
            "sample": "%d full-size rotations (N=2^16, level 24, K=8, dnum=3) of uniform-residue ciphertexts, "
                      "key generation excluded; oracle threads over limbs" % done}


def line_config(world, seeded_a=False):
    """The `config` of the rotation-batch line, identical on both arms."""
    cfg = dict(WORKLOAD, parallelism="replicas%d" % world if world > 1 else "single")
    if seeded_a:
        cfg["keys"] = "seeded a-halves: b stored (0.8 GB per step), a regenerated in the key inner product"
    return cfg


# rotations of the batch that one step of the reference arm times
REF_ROTATIONS_PER_STEP = 2


def run_reference(args, rank, world):
    """The reference arm: the oracle on the host cores, rank 0 only.  Each
    step is a bounded sample of the workload, REF_ROTATIONS_PER_STEP of its 64
    rotations (in batch order), timed with the host clock; value is the
    rotations timed over the time they took, ms_per_step the time of one
    such step."""
    if rank != 0:
        return
    t0 = time.perf_counter()
    o = OracleRotations()
    R = REF_ROTATIONS_PER_STEP
    for i in range(R * (args.warmup + args.steps)):  # keys outside the timing
        o.key(o.ct_steps[i % N_CTS])
    i = 0
    for _ in range(args.warmup):
        for _ in range(R):
            o.rotate(i)
            i += 1
    t_steps = []
    for _ in range(args.steps):
        t = 0.0
        for _ in range(R):
            t += o.rotate(i)
            i += 1
        t_steps.append(t)
    total = float(sum(t_steps))
    v = R * args.steps / total
    sample = ("%d full-size rotations of the batch per step (N=2^16, level 24, K=8, dnum=3), uniform-residue "
              "ciphertexts, key generation excluded; oracle threads over limbs" % R)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "rotations/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps,
            "rotations_per_step": R, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u64", "data": "synthetic", "config": line_config(world),
            "cpu_baseline": {"value": v, "unit": "rotations/s", "cores": o.C.n_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "rotations/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": time.perf_counter() - t0}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ native

def ntt_case(steps, warmup, local_rank, probes=None):
    """The NTT sub-metric: forward and inverse NTT of 512 limbs of 2^16 words
    (256 MiB, larger than L2; 16 polynomials x all 32 primes), device-timed
    per pass.  Butterflies/s per pass against two ceilings: the mixed one
    (integer-path butterflies at the integer probe's rate plus FP64-path
    butterflies at the FP64 probe's rate) and the integer probe's rate alone
    (every butterfly as a 64-bit Shoup product on the integer pipe)."""
    import torch

    from homomorphic_encrypted_transformer_b200 import he

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    ctx = he.he_ctx_create(LOG_N, L, K, DNUM, stream=stream)
    n_polys, n_limbs = 16, L + K
    h = S.uniform_residues(S.master_seed(1), "ntt_residues", ctx.primes, ctx.N, lead=(n_polys,))
    d = torch.from_numpy(h.view(np.int64)).to(dev)
    if probes is None:
        probes = run_probes(he, ctx, dev, stream)
    copy_gbs, int_s, fp_s = probes
    pk, pk_kind = peaks()
    hbm_peak = float(pk.get("hbm_gbs", 6650.0))

    def step():
        he.he_ntt_fwd(ctx, d, n_polys, n_limbs, 0)
        he.he_ntt_inv(ctx, d, n_polys, n_limbs, 0)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    clk = clocks.stop()
    he.he_profile_enable(ctx, True)
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    ok = np.array_equal(d.cpu().numpy().view(np.uint64), h)
    prof = {name: he.he_profile_read(ctx, he.PROF[name]) + (he.he_profile_read_fp(ctx, he.PROF[name]),)
            for name in ("ntt_fwd_cols", "ntt_fwd_rows", "ntt_inv_rows", "ntt_inv_cols")}
    he.he_profile_enable(ctx, False)
    passes = {}
    for name, (pms, n, nbytes, mults, mults_fp) in prof.items():
        if not n:
            continue
        t = pms * 1e-3
        bfly_s = mults / t
        mixed = mults / ((mults - mults_fp) / int_s + mults_fp / fp_s)
        passes[name] = {"us_per_launch": 1e3 * pms / n, "bfly_per_s": bfly_s, "fp64_share": mults_fp / mults,
                        "frac_of_mixed_ceiling": bfly_s / mixed, "frac_of_int_probe": bfly_s / int_s,
                        "hbm_frac": nbytes / t / 1e9 / hbm_peak}
    dom = max(prof, key=lambda k: prof[k][0])
    bfly_step = sum(v[3] for v in prof.values()) / steps
    return {"case": "ntt", "metric": "NTT butterflies/s (N=2^16, 512 limbs: 16 polynomials x 32 primes, forward "
                                     "and inverse)", "value": bfly_step * steps / (ms * 1e-3), "unit": "butterflies/s",
            "ms_per_step": ms / steps, "steps": steps, "warmup": warmup, "roundtrip_ok": bool(ok),
            "roofline": roofline_for(dom, prof[dom], int_s, fp_s, hbm_peak, pk_kind), "passes": passes,
            "probes": {"int_shoup_modmul_per_s": int_s, "fp64_modmul_per_s": fp_s, "copy_gbs": copy_gbs},
            "clocks": clk, "l2": "256 MiB of limbs per transform (larger than L2)"}


def run_rot_small_case(args, local_rank):
    """Kernel case for profiler captures: 8 ciphertexts at level 24 rotated
    with 2 keys (the launch shapes of one key group of the benchmark, ~1 GB)."""
    import torch

    from homomorphic_encrypted_transformer_b200 import he

    torch.cuda.set_device(local_rank)
    ctx = he.he_ctx_create(LOG_N, L, K, DNUM, stream=torch.cuda.current_stream())
    N = ctx.N
    master = S.master_seed(1)
    steps, _ = workload_inputs(master, ctx.primes[:L], N_CTS)
    steps = steps[:2]
    s = S.secret(master, N)
    for st in steps:
        a, e = S.key_draws(master, pow(5, st % (N // 2), 2 * N), ctx.primes, N, DNUM)
        he.he_keygen_upload(ctx, he.HE_KEY_ROTATION, st, s, a, e)
    h = S.uniform_residues(master, "ct_residues", ctx.primes[:L], N, lead=(8, 2))
    x = torch.from_numpy(h.view(np.int64)).cuda()
    y = torch.empty_like(x)
    xs = [he.Ciphertext(x[i], LEVEL, 2.0 ** 40) for i in range(8)]
    ys = [he.Ciphertext(y[i], LEVEL, 2.0 ** 40) for i in range(8)]
    cs = [steps[i % 2] for i in range(8)]
    for _ in range(args.warmup + args.steps):
        he.he_rotate_batch(ctx, xs, cs, ys)
    torch.cuda.synchronize()
    print(json.dumps({"case": "rot_small", "rotations": 8 * (args.warmup + args.steps)}))


def run_ps15_small_case(args, local_rank):
    """Kernel case for profiler captures: the degree-15 evaluation of 8
    ciphertexts at level 24 (the tensor, relinearisation, fused rescale and
    constant-multiply rescale launches of the degree-15 workload at an eighth
    of its batch, ~1.2 GB)."""
    import torch

    from homomorphic_encrypted_transformer_b200 import he

    torch.cuda.set_device(local_rank)
    ctx = he.he_ctx_create(LOG_N, L, K, DNUM, stream=torch.cuda.current_stream())
    N = ctx.N
    master = S.master_seed(4)
    s = S.secret(master, N)
    a, e = S.key_draws(master, 2, ctx.primes, N, DNUM)
    he.he_keygen_upload(ctx, he.HE_KEY_RELIN, 0, s, a, e)
    h = S.uniform_residues(master, "ct_residues", ctx.primes[:L], N, lead=(8, 2))
    x = torch.from_numpy(h.view(np.int64)).cuda()
    y = torch.empty_like(x)
    coeffs = S.poly_coeffs(master, 15)
    xs = [he.Ciphertext(x[i], LEVEL, 2.0 ** 40) for i in range(8)]
    for _ in range(args.warmup + args.steps):
        he.he_poly_eval_ps15(ctx, xs, coeffs, 2.0 ** 62, [he.Ciphertext(y[i], LEVEL, 2.0 ** 40) for i in range(8)])
    torch.cuda.synchronize()
    print(json.dumps({"case": "ps15_small", "evaluations": 8 * (args.warmup + args.steps)}))


# ------------------------------------------------------------------ other workloads

def attention_sum_steps(n_tok, d):
    """Rotation steps the feature sum of he_attention_scores needs (include/he.h):
    2 n b for 0 < b < d1 and 2 n d1 a for 0 < a < d / d1, d1 = 2^ceil(log2(d) / 2)."""
    d1 = 1 << (((d.bit_length() - 1) + 1) // 2)
    return [2 * n_tok * b for b in range(1, d1)] + [2 * n_tok * d1 * a for a in range(1, d // d1)]


FFN = {"n_feat": 256, "n_tok": 128, "bs": 16, "gs": 16, "n_in": 3, "n_out": 12, "level": 12}
# one attention head: d features x n_tok tokens with d 2 n_tok = N/2 at N = 2^16;
# scores shifted by `shift` before the exponential
ATT = {"d": 64, "n_tok": 256, "shift": 1.0}


def device_residues(torch, shape_lead, primes, N, gen, dev):
    """Seeded uniform canonical residues generated on the device:
    [*shape_lead][len(primes)][N] int64 (the kernels' work does not depend on
    the values; parity tests use real encodings and encryptions)."""
    t = torch.empty(tuple(shape_lead) + (len(primes), N), dtype=torch.int64, device=dev)
    for r, q in enumerate(primes):
        t[..., r, :] = torch.randint(0, int(q), tuple(shape_lead) + (N,), dtype=torch.int64, device=dev,
                                     generator=gen)
    return t


def workload_cpu_baseline(case, seconds):
    """The oracle, as it stands, on a bounded sample of a workload (host cores).
    tiny: whole operation sequences at N=2^12.  ps15: whole degree-15
    evaluations of single full-size ciphertexts.  ffn128 / ffn2048: one
    full-size rotation and plaintext products at level 12, timed, scaled by
    the product's operation counts (the key generation is outside every
    timing)."""
    from oracle import ckks as C

    widx = {"tiny": 0, "hoisted": 1, "rotsum": 1, "ffn128": 2, "ffn2048": 3, "ps15": 4, "attention": 5}[case]
    master = S.master_seed(widx)
    t_end = time.perf_counter() + seconds
    if case == "tiny":
        P = C.Params(12, 3, 1, 3)
        s = S.secret(master, P.N)
        keys = {}
        for st in (1, 2, -1):
            a, e = S.key_draws(master, P.galois_elt(st), P.mods, P.N, P.dnum)
            keys[st] = C.rotation_key(s, st, a, e, P)
        a, e = S.key_draws(master, 2, P.mods, P.N, P.dnum)
        rlk = C.relin_key(s, a, e, P)
        ct = C.make_ct(S.uniform_residues(master, "ct_residues", P.q, P.N, lead=(2,)), 3, 2.0 ** 40)
        done, t = 0, 0.0
        while done < 2 or time.perf_counter() < t_end:
            t0 = time.perf_counter()
            C.ntt_rows(C.intt_rows(ct["c"][0], P.q, P), P.q, P)
            for st in (1, 2, -1):
                C.rotate(ct, st, keys[st], P)
            C.hmult_relin_rescale(ct, ct, rlk, P)
            t += time.perf_counter() - t0
            done += 1
        return {"value": done / t, "unit": "sequences/s", "cores": C.n_threads(), "kind": "oracle",
                "sample": "%d whole sequences (NTT round trip, 3 rotations, 1 HMult-relin-rescale), N=2^12" % done}
    P = C.Params(LOG_N, L, K, DNUM)
    s = S.secret(master, P.N)
    if case == "attention":
        d, n_tok = ATT["d"], ATT["n_tok"]
        steps = [1] + sorted({x for st in C.attention_sum_steps(n_tok, d) for x in st if x})
        keys = {}
        for st in steps:
            a, e = S.key_draws(master, P.galois_elt(st), P.mods, P.N, P.dnum)
            keys[st] = C.rotation_key(s, st, a, e, P)
        a, e = S.key_draws(master, 2, P.mods, P.N, P.dnum)
        rlk = C.relin_key(s, a, e, P)
        q, k, v = (C.make_ct(S.uniform_residues(master, "ct_residues", P.q, P.N, i, lead=(2,)), L, 2.0 ** 40)
                   for i in range(3))
        exp_c = [1.0 / math.factorial(j) for j in range(16)]
        done, t = 0, 0.0
        while done < 1 or time.perf_counter() < t_end:
            t0 = time.perf_counter()
            sc = C.attention_scores(q, k, n_tok, d, [1], keys, rlk, P)
            a_ = [C.ps_eval_deg15(x, exp_c, rlk, P) for x in sc]
            C.attention_av(a_, v, [1], keys, rlk, P)
            t += time.perf_counter() - t0
            done += 1
        return {"value": done / (t * n_tok), "unit": "heads/s", "cores": C.n_threads(), "kind": "oracle",
                "sample": "%d full-size token offsets of one head (scores, exponential, output at level 24), "
                          "scaled to the head's %d offsets; key generation excluded" % (done, n_tok)}
    if case in ("hoisted", "rotsum"):
        steps = workload_inputs(master, P.q, N_CTS)[0][:2]
        keys = {}
        for st in steps:
            a, e = S.key_draws(master, P.galois_elt(st), P.mods, P.N, P.dnum)
            keys[st] = C.rotation_key(s, st, a, e, P)
        ct = C.make_ct(S.uniform_residues(master, "ct_residues", P.q, P.N, lead=(2,)), L, 2.0 ** 40)
        done, t = 0, 0.0
        while done < 2 or time.perf_counter() < t_end:
            t0 = time.perf_counter()
            if case == "hoisted":
                C.rotate_hoisted(ct, steps, keys, P)
            else:
                C.rotate_sum_hoisted(ct, steps, keys, P)
            t += time.perf_counter() - t0
            done += len(steps)
        what = "hoisted rotations" if case == "hoisted" else "rotations summed with one ModUp and one ModDown"
        return {"value": done / t, "unit": "rotations/s", "cores": C.n_threads(), "kind": "oracle",
                "sample": "%d full-size %s (level 24), one ciphertext by 2 steps per call; key generation "
                          "excluded" % (done, what)}
    if case == "ps15":
        a, e = S.key_draws(master, 2, P.mods, P.N, P.dnum)
        rlk = C.relin_key(s, a, e, P)
        coeffs = S.poly_coeffs(master, 15)
        ct = C.make_ct(S.uniform_residues(master, "ct_residues", P.q, P.N, lead=(2,)), L, 2.0 ** 40)
        done, t = 0, 0.0
        while done < 1 or time.perf_counter() < t_end:
            t0 = time.perf_counter()
            C.ps_eval_deg15(ct, coeffs, rlk, P)
            t += time.perf_counter() - t0
            done += 1
        return {"value": done / t, "unit": "evals/s", "cores": C.n_threads(), "kind": "oracle",
                "sample": "%d whole degree-15 evaluations of single full-size ciphertexts (level 24)" % done}
    f = FFN
    n_groups = 1 if case == "ffn128" else 16
    lvl = f["level"]
    st = f["n_tok"]
    a, e = S.key_draws(master, P.galois_elt(st), P.mods, P.N, P.dnum)
    key = C.rotation_key(s, st, a, e, P)
    ct = C.make_ct(S.uniform_residues(master, "ct_residues", P.q[:lvl], P.N, lead=(2,)), lvl, 2.0 ** 40)
    pt = S.uniform_residues(master, "pt_residues", P.q[:lvl], P.N, lead=(1,))[0]
    t0 = time.perf_counter()
    C.rotate(ct, st, key, P)
    t_rot = time.perf_counter() - t0
    n_pm, t_pm = 0, 0.0
    while n_pm < 4 or time.perf_counter() < t_end:
        t0 = time.perf_counter()
        C.pmult_accum([ct], [pt], lvl, P)
        t_pm += time.perf_counter() - t0
        n_pm += 1
    t0 = time.perf_counter()
    C.rescale(ct, P)
    t_rs = time.perf_counter() - t0
    rot = n_groups * f["n_in"] * (f["bs"] - 1) + n_groups * f["n_out"] * (f["gs"] - 1)
    pms = n_groups * f["n_out"] * f["n_in"] * f["gs"] * f["bs"]
    per_product = rot * t_rot + pms * t_pm / n_pm + n_groups * f["n_out"] * t_rs
    return {"value": 1.0 / per_product, "unit": "products/s", "cores": C.n_threads(), "kind": "oracle",
            "sample": "1 full-size rotation, %d plaintext products and 1 rescale at level 12, scaled to the "
                      "product's %d rotations, %d plaintext products and %d rescales (%.1f s per product)"
                      % (n_pm, rot, pms, n_groups * f["n_out"], per_product)}


def workload_case(case, n_steps, n_warmup, cpu_seconds, local_rank, probes=None, with_cpu=True, seeded_a=False):
    """Throughput of one of the other workloads on one GPU, as a dict:
    ffn128 (FFN1 768->3072, 128 tokens: 3 x 12 blocks by BSGS at level 12),
    ffn2048 (the same product for 16 token groups sharing the weights),
    ps15 (degree-15 Paterson-Stockmeyer on 64 ciphertexts from level 24),
    tiny (N=2^12 NTT round trip, 3 rotations and one HMult-relin-rescale),
    hoisted (4 ciphertexts at level 24 each rotated by the rotation batch's
    16 steps through one ModUp per ciphertext: 64 hoisted rotations),
    rotsum (the same 4 ciphertexts each summed over its 16 rotations with
    one ModUp and one ModDown: 64 rotations into 4 sums),
    rotation (the rotation batch of the headline, for its seeded-a form),
    attention (one encrypted head at level 24: 64 features x 256 tokens, all
    256 token offsets: scores, the degree-15 exponential, A x V).
    Inputs are seeded uniform residues on the device; the rotation and
    relinearisation keys are computed by the library from seeded draws."""
    import torch

    from homomorphic_encrypted_transformer_b200 import he

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    widx = {"tiny": 0, "rotation": 1, "hoisted": 1, "rotsum": 1, "ffn128": 2, "ffn2048": 3, "ps15": 4,
            "attention": 5}[case]
    master = S.master_seed(widx)
    gen = torch.Generator(device=dev)
    gen.manual_seed(master)
    if case == "tiny":
        ctx = he.he_ctx_create(12, 3, 1, 3, stream=stream)
    else:
        ctx = he.he_ctx_create(LOG_N, L, K, DNUM, stream=stream)
    N = ctx.N
    s_key = S.secret(master, N)

    def upload(kind, step):
        kid = 2 if kind == he.HE_KEY_RELIN else pow(5, step % (N // 2), 2 * N)  # Galois elements are odd
        a, e = S.key_draws(master, kid, ctx.primes, N, ctx.dnum)
        he.he_keygen_upload(ctx, kind, step, s_key, a, e)

    def rotation_keys(steps):
        if seeded_a:
            he.he_keygen_seeded_ex(ctx, master, steps, False, he.HE_KEYGEN_SEEDED_A)
        else:
            for st in steps:
                upload(he.HE_KEY_ROTATION, st)

    if case in ("ffn128", "ffn2048"):
        f = FFN
        n_groups = 1 if case == "ffn128" else 16
        lvl = f["level"]
        steps = sorted({f["n_tok"] * b for b in range(1, f["bs"])} |
                       {f["n_tok"] * f["bs"] * g for g in range(1, f["gs"])})
        for st in steps:
            upload(he.HE_KEY_ROTATION, st)
        pt = device_residues(torch, (f["n_out"], f["n_in"], f["gs"], f["bs"]), ctx.primes[:lvl], N, gen, dev)
        x = device_residues(torch, (n_groups * f["n_in"], 2), ctx.primes[:lvl], N, gen, dev)
        y = torch.empty((n_groups * f["n_out"], 2, lvl, N), dtype=torch.int64, device=dev)
        xs = [he.Ciphertext(x[i], lvl, 2.0 ** 40) for i in range(n_groups * f["n_in"])]

        def step():
            ys = [he.Ciphertext(y[i], lvl, 2.0 ** 40) for i in range(n_groups * f["n_out"])]
            he.he_pmult_accum_bsgs(ctx, xs, f["n_in"], pt, 2.0 ** 40, f["n_out"], f["bs"], f["gs"], f["n_tok"],
                                   n_groups, ys)

        metric, unit = ("FFN1 768->3072 products/s (128 tokens)" if n_groups == 1 else
                        "FFN1 768->3072 products/s (2048 tokens, 16 groups)"), "products/s"
        per_step = 1
        cfg = {"workload": case, "N": N, "level": lvl, "tokens": f["n_tok"] * n_groups, "bs": f["bs"], "gs": f["gs"],
               "rotations_per_step": n_groups * f["n_in"] * (f["bs"] - 1) + n_groups * f["n_out"] * (f["gs"] - 1),
               "weights_gb": pt.numel() * 8 / 1e9}
    elif case == "rotation":
        steps, ct_steps = workload_inputs(master, ctx.primes[:L], N_CTS)
        rotation_keys(steps)
        x = device_residues(torch, (N_CTS, 2), ctx.primes[:L], N, gen, dev)
        y = torch.empty_like(x)
        xs = [he.Ciphertext(x[i], L, 2.0 ** 40) for i in range(N_CTS)]
        ys = [he.Ciphertext(y[i], L, 2.0 ** 40) for i in range(N_CTS)]

        def step():
            he.he_rotate_batch(ctx, xs, ct_steps, ys)

        metric, unit, per_step = METRIC, "rotations/s", N_CTS
        cfg = dict(WORKLOAD)
    elif case == "hoisted":
        steps, _ = workload_inputs(master, ctx.primes[:L], N_CTS)
        rotation_keys(steps)
        n_in = N_CTS // N_KEYS
        x = device_residues(torch, (n_in, 2), ctx.primes[:L], N, gen, dev)
        y = torch.empty((n_in * N_KEYS, 2, L, N), dtype=torch.int64, device=dev)
        xs = [he.Ciphertext(x[i], L, 2.0 ** 40) for i in range(n_in)]

        def step():
            ys = [he.Ciphertext(y[i], L, 2.0 ** 40) for i in range(n_in * N_KEYS)]
            he.he_rotate_hoisted(ctx, xs, steps, ys)

        metric, unit, per_step = "hoisted rotations/s (4 ciphertexts x 16 steps, N=2^16, level 24)", "rotations/s", \
            n_in * N_KEYS
        cfg = {"workload": case, "N": N, "L": L, "K": K, "dnum": DNUM, "level": L, "n_ciphertexts": n_in,
               "n_steps": N_KEYS, "l2": "inputs and keys larger than L2 (1.6 GB of keys per step)"}
    elif case == "rotsum":
        steps, _ = workload_inputs(master, ctx.primes[:L], N_CTS)
        rotation_keys(steps)
        n_in = N_CTS // N_KEYS
        x = device_residues(torch, (n_in, 2), ctx.primes[:L], N, gen, dev)
        y = torch.empty_like(x)
        xs = [he.Ciphertext(x[i], L, 2.0 ** 40) for i in range(n_in)]

        def step():
            he.he_rotate_sum_hoisted(ctx, xs, steps, [he.Ciphertext(y[i], L, 2.0 ** 40) for i in range(n_in)])

        metric, unit, per_step = ("summed rotations/s (4 ciphertexts x 16 steps into 4 sums, N=2^16, level 24)",
                                  "rotations/s", n_in * N_KEYS)
        cfg = {"workload": case, "N": N, "L": L, "K": K, "dnum": DNUM, "level": L, "n_ciphertexts": n_in,
               "n_steps": N_KEYS, "l2": "keys larger than L2 (1.6 GB of keys per step)"}
    elif case == "attention":
        d, n_tok = ATT["d"], ATT["n_tok"]
        offsets = list(range(n_tok))
        for st in sorted(set(offsets[1:]) | set(attention_sum_steps(n_tok, d))):
            upload(he.HE_KEY_ROTATION, st)
        upload(he.HE_KEY_RELIN, 0)
        qkv = device_residues(torch, (3, 2), ctx.primes[:L], N, gen, dev)
        q, k, v = (he.Ciphertext(qkv[i], L, 2.0 ** 40) for i in range(3))
        sbuf = torch.empty((n_tok, 2, L, N), dtype=torch.int64, device=dev)
        abuf = torch.empty_like(sbuf)
        obuf = torch.empty((2, L, N), dtype=torch.int64, device=dev)
        exp_c = [1.0 / math.factorial(j) for j in range(16)]

        def step():
            sc = [he.Ciphertext(sbuf[i], L, 2.0 ** 40) for i in range(n_tok)]
            he.he_attention_scores(ctx, q, k, n_tok, d, offsets, sc)
            kk = int(round(-ATT["shift"] * sc[0].scale))
            for x in sc:
                he.he_add_const(ctx, x, kk)
            a = [he.Ciphertext(abuf[i], L, 2.0 ** 40) for i in range(n_tok)]
            he.he_poly_eval_ps15(ctx, sc, exp_c, 2.0 ** 62, a)
            he.he_attention_output(ctx, a, v, n_tok, offsets, he.Ciphertext(obuf, L, 2.0 ** 40))

        metric, unit, per_step = "attention heads/s (64 features x 256 tokens, N=2^16, level 24)", "heads/s", 1
        cfg = {"workload": case, "N": N, "level": L, "d": d, "tokens": n_tok, "offsets": n_tok,
               "ops_per_head": {"hoisted_rotations": 2 * (n_tok - 1), "rotations": n_tok * (d.bit_length() - 1),
                                "hmult_relin_rescale": 2 * n_tok, "degree15_evals": n_tok}}
    elif case == "ps15":
        upload(he.HE_KEY_RELIN, 0)
        n = 64
        coeffs = S.poly_coeffs(master, 15)
        x = device_residues(torch, (n, 2), ctx.primes[:L], N, gen, dev)
        y = torch.empty_like(x)
        xs = [he.Ciphertext(x[i], L, 2.0 ** 40) for i in range(n)]

        def step():
            ys = [he.Ciphertext(y[i], L, 2.0 ** 40) for i in range(n)]
            he.he_poly_eval_ps15(ctx, xs, coeffs, 2.0 ** 62, ys)

        metric, unit, per_step = "degree-15 polynomial evaluations/s (64 ciphertexts, level 24)", "evals/s", n
        cfg = {"workload": case, "N": N, "level": L, "n_ciphertexts": n, "hmrr_per_eval": 3 + 3}
    else:
        for st in (1, 2, -1):
            upload(he.HE_KEY_ROTATION, st)
        upload(he.HE_KEY_RELIN, 0)
        x = device_residues(torch, (2,), ctx.primes, N, gen, dev)[:, :3].contiguous()
        d = device_residues(torch, (1,), ctx.primes[:3], N, gen, dev)
        r = torch.empty_like(x)
        xc = he.Ciphertext(x, 3, 2.0 ** 40)

        def step():
            he.he_ntt_inv(ctx, d, 1, 3, 0)
            he.he_ntt_fwd(ctx, d, 1, 3, 0)
            for st in (1, 2, -1):
                he.he_rotate(ctx, xc, st, he.Ciphertext(r, 3, 2.0 ** 40))
            he.he_hmult_relin_rescale(ctx, xc, xc, he.Ciphertext(r, 3, 2.0 ** 40))

        metric, unit, per_step = "tiny-config operation sequences/s (N=2^12)", "sequences/s", 1
        cfg = {"workload": case, "N": N, "ops": "NTT round trip, 3 rotations, 1 HMult-relin-rescale",
               "l2": "inputs L2-resident (a latency-bound sequence of small launches)"}

    for _ in range(n_warmup):
        step()
    torch.cuda.synchronize()
    copy_gbs, int_modmul_s, fp_modmul_s = probes if probes is not None else run_probes(he, ctx, dev, stream)
    pk, pk_kind = peaks()
    hbm_peak = float(pk.get("hbm_gbs", 6650.0))
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(n_steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    if case == "tiny":
        # launch-bound: the same sequence captured once as a CUDA graph and
        # replayed (the eager calls above sized the scratch); value = replay
        ms_eager = ms
        graph = capture_graph(he, ctx, step, stream)
        graph.replay()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(n_steps):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1)
        del graph
        cfg["cuda_graph"] = "value: one captured sequence replayed per step; eager_value: the calls issued one by one"
        cfg["eager_value"] = per_step * n_steps / (ms_eager * 1e-3)
    clk = clocks.stop()
    he.he_profile_enable(ctx, True)
    for _ in range(n_steps):
        step()
    prof = {name: he.he_profile_read(ctx, cls) + (he.he_profile_read_fp(ctx, cls),) for name, cls in he.PROF.items()}
    he.he_profile_enable(ctx, False)
    dom = max(prof, key=lambda k: prof[k][0])
    alu_ideal = sum(((v[3] - v[4]) / int_modmul_s + v[4] / fp_modmul_s) * 1e3 for v in prof.values()) / n_steps
    line = {"case": case, "metric": metric, "value": per_step * n_steps / (ms * 1e-3), "unit": unit,
            "ms_per_step": ms / n_steps, "steps": n_steps, "warmup": n_warmup, "n_gpus": 1,
            "higher_is_better": True, "dtype": "u64", "data": "synthetic (seeded uniform residues, seeded keys)",
            "config": cfg, "roofline": roofline_for(dom, prof[dom], int_modmul_s, fp_modmul_s, hbm_peak, pk_kind),
            "alu_ideal_ms_per_step": alu_ideal,
            "kernel_ms_per_step": {k: round(v[0] / n_steps, 4) for k, v in prof.items() if v[1]},
            "kernel_roofline_frac": {k: round(roofline_for(k, v, int_modmul_s, fp_modmul_s, hbm_peak,
                                                           pk_kind)["frac"], 3) for k, v in prof.items() if v[1]},
            "probes": {"copy_gbs": copy_gbs, "int_shoup_modmul_per_s": int_modmul_s,
                       "fp64_modmul_per_s": fp_modmul_s},
            "clocks": clk}
    if seeded_a:
        cfg["keys"] = "seeded a-halves: b stored, a regenerated in the key inner product"
    if case == "ps15":
        line["hmrr_per_s"] = line["value"] * cfg["hmrr_per_eval"]
    if with_cpu:
        line["cpu_baseline"] = workload_cpu_baseline(case, cpu_seconds)
    return line


def capture_graph(he, ctx, step, stream):
    """step() captured as one CUDA graph on a side stream (the context's
    calls enqueue there during the capture), for replay on `stream`."""
    import torch

    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    he.he_set_stream(ctx, cap)
    try:
        with torch.cuda.stream(cap):
            g.capture_begin()
            try:
                step()
            finally:
                g.capture_end()
    finally:
        he.he_set_stream(ctx, stream)
    stream.wait_stream(cap)
    return g


# the other workloads of the default run: (warm-up steps, timed steps) each.
# A name ending in _seeded_a is its workload with seeded a-halves in every
# key (HE_KEYGEN_SEEDED_A); its oracle baseline is the stored-key entry's
# (the oracle's work does not depend on how the key is kept).
WORKLOAD_STEPS = {"ntt": (3, 10), "tiny": (3, 20), "hoisted": (3, 10), "rotsum": (3, 10), "ps15": (3, 5),
                  "ffn128": (3, 4), "ffn2048": (3, 2), "attention": (3, 2), "rotation_seeded_a": (3, 10),
                  "hoisted_seeded_a": (3, 10)}
SEEDED_A_SUFFIX = "_seeded_a"
# seconds of oracle work per workload's cpu_baseline in the default run
WORKLOAD_CPU_SECONDS = 3.0


def all_workloads(local_rank, probes):
    """Every other workload, one after the other in this process, as
    {case: dict}; each frees its device memory before the next."""
    import gc

    import torch

    out = {}
    for case, (w, k) in WORKLOAD_STEPS.items():
        t0 = time.perf_counter()
        if case == "ntt":
            r = ntt_case(k, w, local_rank, probes)
        elif case.endswith(SEEDED_A_SUFFIX):
            r = workload_case(case[:-len(SEEDED_A_SUFFIX)], k, w, WORKLOAD_CPU_SECONDS, local_rank, probes,
                              with_cpu=False, seeded_a=True)
        else:
            r = workload_case(case, k, w, WORKLOAD_CPU_SECONDS, local_rank, probes)
        r["wall_s"] = time.perf_counter() - t0
        out[case] = r
        gc.collect()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def run_probes(he, ctx, dev, stream):
    """HBM copy, integer and FP64 modular-product probes in the same run:
    (copy GB/s, integer products/s, FP64 products/s)."""
    import torch

    probe_words = 1 << 28  # 2 GiB each way
    pa = torch.empty(probe_words, dtype=torch.int64, device=dev)
    pb = torch.empty_like(pa)
    pa.fill_(1)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = 1e9
    for _ in range(5):
        ev0.record(stream)
        he.he_probe_copy(ctx, pb, pa, probe_words)
        ev1.record(stream)
        torch.cuda.synchronize()
        best = min(best, ev0.elapsed_time(ev1))
    copy_gbs = 2 * probe_words * 8 / (best * 1e-3) / 1e9
    del pa, pb
    sink = torch.empty(he.he_probe_int_threads(ctx), dtype=torch.int64, device=dev)
    iters = 4096
    rates = []
    for fn in (he.he_probe_int, he.he_probe_fp):
        best = 1e9
        for _ in range(3):
            ev0.record(stream)
            fn(ctx, iters, sink)
            ev1.record(stream)
            torch.cuda.synchronize()
            best = min(best, ev0.elapsed_time(ev1))
        rates.append(he.he_probe_int_threads(ctx) * iters * he.he_probe_int_mults_per_iter() / (best * 1e-3))
    return copy_gbs, rates[0], rates[1]


def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from homomorphic_encrypted_transformer_b200 import he

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    ctx = he.he_ctx_create(LOG_N, L, K, DNUM, stream=stream)
    N = ctx.N
    master = S.master_seed(1)
    steps, ct_steps = workload_inputs(master, ctx.primes[:L], N_CTS)
    if args.seeded_a:
        he.he_keygen_seeded_ex(ctx, master, steps, False, he.HE_KEYGEN_SEEDED_A)
    else:
        s = S.secret(master, N)
        for st in steps:
            k = pow(5, st % (N // 2), 2 * N)
            a, e = S.key_draws(master, k, ctx.primes, N, DNUM)
            he.he_keygen_upload(ctx, he.HE_KEY_ROTATION, st, s, a, e)
    # inputs: uniform residues (a fresh encryption is computationally
    # indistinguishable from them); per-rank stream of draws
    h_in = S.uniform_residues(rank_seed(master, rank), "ct_residues", ctx.primes[:L], N, lead=(N_CTS, 2))
    x = torch.from_numpy(h_in.view(np.int64)).to(dev)
    y = torch.empty_like(x)
    xs = [he.Ciphertext(x[i], LEVEL, 2.0 ** 40) for i in range(N_CTS)]
    ys = [he.Ciphertext(y[i], LEVEL, 2.0 ** 40) for i in range(N_CTS)]

    def step():
        he.he_rotate_batch(ctx, xs, ct_steps, ys)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    copy_gbs, int_modmul_s, fp_modmul_s = run_probes(he, ctx, dev, stream)

    # timed region (the headline number): K steps, no profiling events
    clocks = ClockSampler(local_rank)
    he.he_launch_count(ctx, reset=True)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_plain = t0.elapsed_time(t1)
    clk = clocks.stop()
    launches = he.he_launch_count(ctx)

    # the same steps again with every launch class bracketed by events on the
    # launching stream: per-kernel device time and algorithmic work
    he.he_profile_enable(ctx, True)
    torch.cuda.synchronize()
    barrier()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1)
    prof = {name: he.he_profile_read(ctx, cls) + (he.he_profile_read_fp(ctx, cls),) for name, cls in he.PROF.items()}
    he.he_profile_enable(ctx, False)

    ms_plain, ms = max_over_ranks([ms_plain, ms], world, dev)

    # end to end through the host-buffer entry points (pinned host memory):
    # the ciphertexts in the packed wire format (he_rotate_batch_host_wire,
    # the e2e figure) and as 64-bit words (he_rotate_batch_host)
    e2e_steps = max(1, min(args.steps, 5))
    w_in = torch.from_numpy(he.he_ct_pack(ctx.primes, LEVEL, LOG_N, h_in)).pin_memory()
    w_out = torch.empty_like(w_in).pin_memory()
    he.he_rotate_batch_host_wire(ctx, w_in, LEVEL, ct_steps, w_out)
    barrier()
    te = time.perf_counter()
    for _ in range(e2e_steps):
        he.he_rotate_batch_host_wire(ctx, w_in, LEVEL, ct_steps, w_out)
    e2e_s = time.perf_counter() - te
    h_pin = torch.from_numpy(h_in.view(np.int64)).pin_memory()
    h_out = torch.empty_like(h_pin).pin_memory()
    he.he_rotate_batch_host(ctx, h_pin, LEVEL, ct_steps, h_out)
    barrier()
    te = time.perf_counter()
    for _ in range(e2e_steps):
        he.he_rotate_batch_host(ctx, h_pin, LEVEL, ct_steps, h_out)
    e2e_words_s = time.perf_counter() - te
    e2e_s, e2e_words_s = max_over_ranks([e2e_s, e2e_words_s], world, dev)

    if rank != 0:
        return None
    total_rot = N_CTS * args.steps * world
    value = total_rot / (ms_plain * 1e-3)
    pk, pk_kind = peaks()
    hbm_peak = float(pk.get("hbm_gbs", 6650.0))
    # dominant kernel class by device time in the profiled pass
    dom_name = max(prof, key=lambda k: prof[k][0])
    ct_bytes = 2 * LEVEL * N * 8
    key_bytes = 3 * (1 if args.seeded_a else 2) * (L + K) * N * 8  # digits x stored halves x rows
    # algorithmic bytes of one rotation batch (keys read once per key group)
    batch_bytes = N_KEYS * key_bytes + N_CTS * 2 * ct_bytes
    hbm_frac_step = (batch_bytes / (ms_plain * 1e-3 / args.steps)) / 1e9 / hbm_peak
    roof = roofline_for(dom_name, prof[dom_name], int_modmul_s, fp_modmul_s, hbm_peak, pk_kind)
    # ideal time of a whole step: each class's modular products at the probes'
    # rates (integer and FP64 pipes taken one after the other)
    alu_ideal_ms = sum(((v[3] - v[4]) / int_modmul_s + v[4] / fp_modmul_s) * 1e3 for v in prof.values()) / args.steps
    line = {"metric": METRIC, "value": value, "unit": "rotations/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_plain / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u64", "data": "synthetic",
            "config": line_config(world, args.seeded_a),
            "hbm_roofline_frac_of_step": hbm_frac_step,
            # the same with every rotation reading its own key (no reuse across the batch)
            "hbm_roofline_frac_no_key_reuse": (N_CTS * (key_bytes + 2 * ct_bytes) / (ms_plain * 1e-3 / args.steps))
            / 1e9 / hbm_peak,
            "alu_ideal_ms_per_step": alu_ideal_ms,
            "alu_roofline_frac_of_step": alu_ideal_ms / (ms_plain / args.steps),
            "roofline": roof,
            "probes": {"copy_gbs": copy_gbs, "int_shoup_modmul_per_s": int_modmul_s,
                       "fp64_modmul_per_s": fp_modmul_s},
            "kernel_ms_per_step": {k: round(v[0] / args.steps, 4) for k, v in prof.items() if v[1]},
            "kernel_launches_per_step": {k: v[1] / args.steps for k, v in prof.items() if v[1]},
            "kernel_roofline_frac": {k: round(roofline_for(k, v, int_modmul_s, fp_modmul_s, hbm_peak,
                                                           pk_kind)["frac"], 3)
                                     for k, v in prof.items() if v[1]},
            "profiled_ms_per_step": ms / args.steps,
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": {"value": N_CTS * e2e_steps * world / e2e_s, "unit": "rotations/s",
                    "h2d_bytes_per_step": int(w_in.numel()), "d2h_bytes_per_step": int(w_out.numel()),
                    "format": "packed wire format: 5 bytes per 40-bit residue, 8 per 60-bit (he_ct_pack)",
                    "words": {"value": N_CTS * e2e_steps * world / e2e_words_s, "unit": "rotations/s",
                              "h2d_bytes_per_step": int(h_in.nbytes), "d2h_bytes_per_step": int(h_in.nbytes),
                              "format": "64-bit words (he_rotate_batch_host)"}}}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    line["_probes"] = (copy_gbs, int_modmul_s, fp_modmul_s)
    return line


# ncu DRAM bytes (read + write) of one launch over that launch's algorithmic
# bytes, per kernel class, from one capture of the kernel.  `sources` are the
# files the kernel is built from and `sha256` their digest (source_digest)
# when the counters were taken: a ratio whose sources have changed since is
# not used, and `traffic` is then null.  Reads grow in proportion to the limbs
# a launch transforms; a small capture leaves some written lines in L2 at its
# end, so the ratio slightly undercounts writes.
NTT_SOURCES = ["homomorphic_encrypted_transformer_b200/csrc/ntt.cu", "homomorphic_encrypted_transformer_b200/csrc/ntt.cuh",
               "homomorphic_encrypted_transformer_b200/csrc/modarith.cuh",
               "homomorphic_encrypted_transformer_b200/csrc/kernels.cuh"]
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of the four
# transform passes on 512 limbs of 2^16 words (bench.py --case ntt; each pass
# reads and writes 268.4 MB of limbs), taken with the sources of this digest
NTT_SHA256 = "0eeb6e0dc51e6a7f1939d8cfd007c567a91aea1a08579ff357f1f62e1633ac71"
NCU_TRAFFIC = {
    "ntt_fwd_cols": {"ratio": (268579072 + 218044416) / 536870912.0, "sources": NTT_SOURCES, "sha256": NTT_SHA256},
    "ntt_fwd_rows": {"ratio": (311915776 + 216503296) / 536870912.0, "sources": NTT_SOURCES, "sha256": NTT_SHA256},
    "ntt_inv_rows": {"ratio": (313877760 + 213612800) / 536870912.0, "sources": NTT_SOURCES, "sha256": NTT_SHA256},
    "ntt_inv_cols": {"ratio": (268575744 + 214055424) / 536870912.0, "sources": NTT_SOURCES, "sha256": NTT_SHA256},
}


def source_digest(files):
    """sha256 over the named repository files (path and contents, in order)."""
    import hashlib

    h = hashlib.sha256()
    for f in files:
        h.update(f.encode())
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_ratio(name, table=None):
    """The stored ncu traffic ratio of a kernel class, or None when there is
    none or its sources changed after the capture."""
    e = (NCU_TRAFFIC if table is None else table).get(name)
    if not e:
        return None
    try:
        if source_digest(e["sources"]) != e["sha256"]:
            return None
    except OSError:
        return None
    return e["ratio"]


def roofline_for(name, prof_entry, int_modmul_s, fp_modmul_s, hbm_peak, pk_kind):
    """Roofline of the dominant kernel class: its algorithmic bytes and
    modular multiplications per launch (counted by the library as it
    launches, split between the integer and the FP64 pipe) against its
    CUDA-event duration.  The ALU ceiling of the class is the time its
    products take at the two probes' rates (integer products at the integer
    probe's rate, FP64 products at the FP64 probe's); the binding resource is
    the one whose ideal time is longer."""
    ms, launches, nbytes, mults, mults_fp = prof_entry
    launches = max(1, launches)
    t = ms * 1e-3 / launches
    b, m, m_fp = nbytes / launches, mults / launches, mults_fp / launches
    t_hbm = b / (hbm_peak * 1e9)
    t_alu = (m - m_fp) / int_modmul_s + (m_fp / fp_modmul_s if fp_modmul_s > 0 else 0.0)
    ratio = traffic_ratio(name)
    traffic = ratio * b if ratio is not None else None
    if t_hbm >= t_alu:
        ach = b / t / 1e9
        return {"kernel": name, "bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                "frac": ach / hbm_peak, "traffic": traffic, "algorithmic_bytes_per_launch": b,
                "ms_per_launch": t * 1e3, "peak_source": pk_kind + " (MEASURED_PEAKS.json hbm_gbs)"}
    ach = m / t / 1e9
    peak = m / t_alu / 1e9
    return {"kernel": name, "bound": "alu", "achieved": ach, "peak": peak, "unit": "Gmodmul/s",
            "frac": ach / peak, "traffic": traffic, "algorithmic_modmuls_per_launch": m,
            "fp64_share": m_fp / m if m else 0.0,
            "algorithmic_bytes_per_launch": b, "ms_per_launch": t * 1e3,
            "hbm_frac": (b / t / 1e9) / hbm_peak,
            "peak_source": "in-run probes (register-only modular products over a full grid): integer Shoup "
                           "%.0f G/s, FP64 rounded-quotient %.0f G/s, weighted by this class's mix"
                           % (int_modmul_s / 1e9, fp_modmul_s / 1e9)}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        backend = "nccl" if args.impl == "native" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.case == "ntt":
            print(json.dumps(ntt_case(args.steps, args.warmup, local_rank)), flush=True)
        elif args.case == "rot_small":
            run_rot_small_case(args, local_rank)
        elif args.case == "ps15_small":
            run_ps15_small_case(args, local_rank)
        elif args.case in ("ffn128", "ffn2048", "ps15", "tiny", "hoisted", "rotsum", "attention"):
            print(json.dumps(workload_case(args.case, args.steps, args.warmup, args.cpu_seconds, local_rank,
                                           with_cpu=not args.no_cpu_baseline, seeded_a=args.seeded_a)), flush=True)
        else:
            line = run_native(args, rank, world, local_rank)
            if line is not None:
                probes = line.pop("_probes")
                # the other workloads on one GPU (the scaling runs time the
                # rotation batch alone)
                if world == 1 and not args.no_workloads:
                    line["workloads"] = all_workloads(local_rank, probes)
                print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
