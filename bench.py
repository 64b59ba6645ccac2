#!/usr/bin/env python
"""Benchmark of the H-BitLinear forward pass (BitNet v2) on B200.

Workload (one step = one pass of the whole layer over one batch):
  ffn_wdown: X bf16 [8192 x 16384] (silu(a)*b, 1% outlier channels x40) ->
  RMSNorm -> online Hadamard transform -> INT4 absmean codes -> ternary matmul
  with W [4096 x 16384] (2-bit packed, absmean) -> bf16 Y [8192 x 4096].
The packed weights are made once (offline step, not timed).

Prints one JSON line (rank 0).  `value` is device-timed tokens/s with inputs
resident in HBM (inputs larger than L2); `e2e` is the same metric through the
host-buffer C-ABI call with the host<->device copies inside the timed region.
`roofline` covers the dominant kernel, timed live with CUDA events on its
stream; `quant` reports the fused norm+transform+quantisation kernel on the
8192 x 4096 workload in GB/s against the measured HBM copy bandwidth.
Multi-GPU (torchrun): every rank runs its own 8192-token batch with a replica
of the packed weights (rows shard with no collective), weak scaling; times
are the max over ranks.

--impl reference times the CPU oracle (the plain scalar C statement of the
layer, test infrastructure) on a bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "H-BitLinear tokens/s (7B W_down, a4) & FWHT+quant GB/s, % roofline"
UNIT = "tokens/s"
M_TOK, K_IN, N_OUT, BITS = 8192, 16384, 4096, 4
QM, QK = 8192, 4096  # quant workload
WORKLOAD = "ffn_wdown: X bf16 [8192 x 16384] -> Y bf16 [8192 x 4096], INT4 absmean act, " \
           "ternary W [4096 x 16384] 2-bit packed"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hbl", choices=["hbl", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-iters", type=int, default=200,
                    help="iterations of the per-kernel timing loops")
    ap.add_argument("--only", default=None,
                    choices=["forward", "gemm", "quant4", "quant8", "nohad4", "ln4", "rotate",
                             "kv3", "kv4", "kv8", "decode_wo", "decode_wdown", "decode_wdown_t32",
                             "decode_wo_t32", "gemv_rows", "gemv_splitk", "pack", "expand",
                             "int8_probe", "gemm_packed", "gemm_pair"],
                    help="run only this case (a few launches, for profiler captures); prints a "
                         "short JSON line, not the benchmark line")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


SM_MAX_MHZ = 1965.0  # B200 clocks.max.sm


def fp32_view(elements, L, t, sms, clock_mhz):
    """K1 against the FP32 lanes instead of HBM: per element L butterfly
    add/subs, the square and its tree add, the products by 1/rms and 1/sqrt(K),
    the |v| (or max) tree step and the quantising FMA = L + 6 operations; peak =
    SMs x 128 FP32 lanes x the maximum SM clock."""
    ops = float(elements) * (L + 6)
    peak = sms * 128 * clock_mhz * 1e6 / 1e12
    ach = ops / t / 1e12
    return {"bound": "alu", "unit": "Tops/s (fp32)", "ops": ops, "achieved": ach, "peak": peak,
            "frac": ach / peak, "peak_note": "%d SMs x 128 fp32 lanes x %.0f MHz" % (sms, clock_mhz)}


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="hbl_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        res = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return res
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if sm:
            res = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                   "reasons": sorted(reasons), "samples": len(sm)}
        return res


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "hadamard_rotated_int4_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key, src_hash):
    """DRAM bytes per launch from a committed ncu capture, if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != src_hash:
        return None
    return e.get("dram_bytes_per_launch")


def cpu_baseline(X_bits, packed, alpha, target_s=15.0):
    """The oracle, as it stands, on a bounded sample of the workload's rows."""
    import numpy as np

    import oracle

    threads = os.cpu_count() or 1
    rows = min(threads, 64)
    while True:  # grow the sample until it takes about target_s (or covers the workload)
        t0 = time.perf_counter()
        oracle.hbitlinear_forward(X_bits[:rows], packed, alpha, BITS, threads=threads)
        dt = time.perf_counter() - t0
        if dt >= target_s / 2 or rows >= M_TOK:
            break
        rows = min(M_TOK, max(rows * 2, int(rows * target_s / max(dt, 1e-3))))
    used = min(threads, rows)
    # the same oracle on one core, a few rows (a second figure for scale)
    r1 = 2
    t1 = time.perf_counter()
    oracle.hbitlinear_forward(X_bits[:r1], packed, alpha, BITS, threads=1)
    d1 = time.perf_counter() - t1
    return {"value": rows / dt, "unit": UNIT, "cores": used, "kind": "oracle",
            "value_1core": r1 / d1, "cpu_model": cpu_model(),
            "sample": "%d of the 8192 token rows of the ffn_wdown workload (full K, full N), "
                      "scalar C oracle, rows split over %d threads, %.1f s; value_1core: %d rows "
                      "on one thread, %.1f s" % (rows, used, dt, r1, d1)}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    from hadamard_rotated_int4_b200 import inputs

    X = inputs.activations("ffn_wdown")
    W = inputs.weights("ffn_wdown")
    packed, alpha = oracle.pack_ternary(W)
    threads = os.cpu_count() or 1
    # 4 token rows per thread per step (the oracle unpacks the weights once per
    # call, shared by its threads), so a step times the oracle's arithmetic
    rows_per_step = min(8192, 4 * max(1, threads))
    for i in range(args.warmup):
        oracle.hbitlinear_forward(X[i * rows_per_step:(i + 1) * rows_per_step], packed, alpha,
                                  BITS, threads=threads)
    t0 = time.perf_counter()
    for i in range(args.steps):
        lo = (i * rows_per_step) % (M_TOK - rows_per_step + 1)
        oracle.hbitlinear_forward(X[lo:lo + rows_per_step], packed, alpha, BITS, threads=threads)
    dt = time.perf_counter() - t0
    value = args.steps * rows_per_step / dt
    used = min(threads, rows_per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_TOK, "K": K_IN, "N": N_OUT, "act_bits": BITS,
                   "global_batch": args.gpus * M_TOK,
                   "parallelism": "replicas by token rows (no collective)" if args.gpus > 1
                   else "single GPU",
                   "l2": "inputs larger than L2 (X 268 MB per step)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": "each step: %d token rows of the ffn_wdown workload (full K "
                                   "and N), scalar C oracle over %d threads (%d rows each)"
                                   % (rows_per_step, used, -(-rows_per_step // used))},
        "rows_per_step": rows_per_step,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def run_hbl(args):
    import numpy as np
    import torch

    import hadamard_rotated_int4_b200 as hbl
    from hadamard_rotated_int4_b200 import dist as hdist
    from hadamard_rotated_int4_b200 import inputs

    rank, local_rank, world = hdist.env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    pk = peaks()
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    # ---- inputs: each rank its own 8192-token batch; the same weights everywhere
    X_bits = inputs.activations("ffn_wdown", seed=rank)
    W = inputs.weights("ffn_wdown")
    Xd = torch.from_numpy(X_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    packed, alpha = hbl.pack_ternary(torch.from_numpy(W).to(dev))
    ws = torch.empty(hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, M_TOK, K_IN, N_OUT, BITS),
                     dtype=torch.uint8, device=dev)
    Y = torch.empty((M_TOK, N_OUT), dtype=torch.bfloat16, device=dev)
    status = hbl.new_status(dev)
    stream = torch.cuda.current_stream()

    def step():
        hbl.hbitlinear_forward(Xd, packed, alpha, BITS, ws=ws, out=Y, status=status)

    sampler = ClockSampler(local_rank)
    for _ in range(max(3, args.warmup)):
        step()
    barrier()
    sampler.start()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    t_dev_ms = e0.elapsed_time(e1)
    t_max_ms = hdist.max_over_ranks(t_dev_ms, dev)
    value = world * M_TOK * args.steps / (t_max_ms / 1e3)

    # ---- per-kernel timing: the forward's stages as separate C-ABI calls with
    # the layouts the fused forward uses at this batch (one-byte INT4 codes for
    # the TMA-fed GEMM; the packed weights expanded to signed bytes per call --
    # the forward itself widens them inside its quantiser at this shape)
    B8 = hbl.ACT_INT4_BYTES
    codes = torch.empty(hbl.codes_shape(M_TOK, K_IN, B8), dtype=torch.uint8, device=dev)
    scales = torch.empty(M_TOK, dtype=torch.float32, device=dev)
    rowsum = torch.empty(M_TOK, dtype=torch.int32, device=dev)
    Ws = torch.empty((N_OUT, K_IN), dtype=torch.int8, device=dev)
    iters = max(args.kernel_iters, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(iters)]
    for i in range(3):
        hbl.norm_fwht_quant(Xd, B8, out=(codes, scales, rowsum))
        hbl.expand_ternary(packed, K_IN, out=Ws)
        hbl.ternary_gemm_s8w(codes, scales, B8, Ws, alpha, out=Y)
    torch.cuda.synchronize()
    for i in range(iters):
        evs[i][0].record(stream)
        hbl.norm_fwht_quant(Xd, B8, out=(codes, scales, rowsum))
        evs[i][1].record(stream)
        hbl.expand_ternary(packed, K_IN, out=Ws)
        evs[i][2].record(stream)
        hbl.ternary_gemm_s8w(codes, scales, B8, Ws, alpha, out=Y, status=status)
        evs[i][3].record(stream)
    torch.cuda.synchronize()
    t_k1 = statistics.mean(e[0].elapsed_time(e[1]) for e in evs) * 1e-3
    t_kx = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) * 1e-3
    t_k2 = statistics.mean(e[2].elapsed_time(e[3]) for e in evs) * 1e-3
    del Ws

    # ---- dense INT8 tensor-core rate of this GPU (the GEMM's roofline denominator)
    probe_mmas = 1 << 15
    probe_tops, probe_st = hbl.measure_int8_tensor_peak(n_sms, probe_mmas, reps=5)
    int8_probe = {"tops": probe_tops, "mmas_per_cta": probe_mmas, "ctas": n_sms,
                  "status": probe_st}

    # Device time per call of a short kernel: `iters` calls (cycling over n
    # inputs) captured in one CUDA graph and replayed, CUDA events around the
    # replays on this stream, so the host's per-call cost stays out of it.
    def graph_time(fn, n, iters, reps=5):
        for i in range(3):
            fn(i % n)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(iters):
                    fn(i % n)
        stream.wait_stream(side)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) * 1e-3 / (reps * iters)

    # ---- quant workload: 8192 x 4096, a4 and a8, 4 rotating inputs (256 MB > L2)
    qX = [torch.from_numpy(inputs.activations("quant", seed=s).view(np.int16)).view(
        torch.bfloat16).to(dev) for s in range(4)]
    quant = {}
    for bits in (4, 8):
        qc = torch.empty((QM, QK if bits == 8 else QK // 2), dtype=torch.uint8, device=dev)
        qs = torch.empty(QM, dtype=torch.float32, device=dev)
        qr = torch.empty(QM, dtype=torch.int32, device=dev)
        t = graph_time(lambda i: hbl.norm_fwht_quant(qX[i], bits, out=(qc, qs, qr)), 4,
                       max(args.kernel_iters, 40))
        nbytes = QM * QK * 2 + QM * QK * bits // 8 + QM * 4 + QM * 4
        gbs = nbytes / t / 1e9
        quant["a%d" % bits] = {"workload": "quant 8192 x 4096 Student-t nu=3, 1% channels x20",
                               "us": t * 1e6, "bytes": nbytes, "achieved_gbs": gbs,
                               "frac": gbs / pk["hbm_gbs"],
                               "alu_view": fp32_view(QM * QK, 12, t, n_sms, SM_MAX_MHZ)}
    del qX

    # ---- decode-batch sweep: T tokens through the whole layer, Wo 4096x4096 and
    # W_down 4096x16384; weight copies rotate so the packed weights (4.2 / 16.8 MB)
    # come from HBM (copies total > 2x L2)
    decode = []
    for shape, Kd in (("wo", 4096), ("wdown", 16384)):
        Wd = torch.from_numpy(inputs.latent_weights(N_OUT, Kd, seed=7)).to(dev)
        p0, a0 = hbl.pack_ternary(Wd)
        del Wd
        ncopy = max(2, int(2.2 * 126e6 // (N_OUT * Kd // 4)) + 1)
        pcs = [p0.clone() for _ in range(ncopy)]
        for T in inputs.DECODE_TOKENS:
            Xt = torch.from_numpy(inputs.activations("decode_" + shape, M=T, K=Kd, seed=T).view(
                np.int16)).view(torch.bfloat16).to(dev)
            wsd = torch.empty(max(16, hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, T, Kd, N_OUT,
                                                         BITS)), dtype=torch.uint8, device=dev)
            Yt = torch.empty((T, N_OUT), dtype=torch.bfloat16, device=dev)
            for i in range(5):
                hbl.hbitlinear_forward(Xt, pcs[i % ncopy], a0, BITS, ws=wsd, out=Yt)
            torch.cuda.synchronize()
            # one CUDA graph holds one forward per weight copy; replays remove the
            # host launch cost that would otherwise dominate a decode step
            graph = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream()
            cap.wait_stream(stream)
            with torch.cuda.stream(cap):
                with torch.cuda.graph(graph, stream=cap):
                    for i in range(ncopy):
                        hbl.hbitlinear_forward(Xt, pcs[i], a0, BITS, ws=wsd, out=Yt)
            stream.wait_stream(cap)
            graph.replay()
            torch.cuda.synchronize()
            reps = max(3, 400 // ncopy)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                graph.replay()
            b.record(stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(b) * 1e-3 / (reps * ncopy)
            del graph
            wbytes = N_OUT * Kd // 4
            decode.append({"shape": shape, "T": T, "K": Kd, "N": N_OUT, "us": t * 1e6,
                           "tokens_per_s": T / t, "packed_w_gbs": wbytes / t / 1e9,
                           "frac_hbm_on_packed_w": wbytes / t / 1e9 / pk["hbm_gbs"],
                           "path": ("one kernel (quantiser in every CTA, weights by bulk copy)"
                                    if T <= 16384 // Kd
                                    else "K1 + GEMV half of the one-kernel forward (weights "
                                         "bulk-copied under K1)"
                                    if Kd == 16384 and T <= 4
                                    else "row GEMV (weight rows per warp, PDL after K1)"
                                    if T <= 4
                                    else "K1 + decode tensor-core kernel (weights in TMEM as "
                                         "A, tokens as B, cluster K-split, DSMEM reduction)"
                                    if T <= 64 or (T <= 128 and Kd <= 8192)
                                    else "gemm_ts (TMEM activations, one-wave split-K)"),
                           "timing": "CUDA graph replay, one forward per weight copy"})
        del pcs

    # ---- the other rows of the hot path, each against the HBM roofline
    ev_time = graph_time

    others = {}
    # BitLinear variants (no Hadamard / LayerNorm) on the quant workload, a4 packed
    qX = [torch.from_numpy(inputs.activations("quant", seed=s).view(np.int16)).view(
        torch.bfloat16).to(dev) for s in range(4)]
    qc = torch.empty((QM, QK // 2), dtype=torch.uint8, device=dev)
    qs = torch.empty(QM, dtype=torch.float32, device=dev)
    qr = torch.empty(QM, dtype=torch.int32, device=dev)
    for name, fl in (("no_hadamard", hbl.NORM_NO_HADAMARD), ("layernorm", hbl.NORM_LAYERNORM),
                     ("layernorm_no_hadamard", hbl.NORM_LAYERNORM | hbl.NORM_NO_HADAMARD)):
        t = ev_time(lambda i: hbl.norm_quant(qX[i], 4, fl, out=(qc, qs, qr)), 4, 40)
        nbytes = QM * QK * 2 + QM * QK // 2 + 8 * QM
        others["norm_quant_a4_" + name] = {
            "workload": "quant 8192 x 4096, a4 packed", "us": t * 1e6, "bytes": nbytes,
            "achieved_gbs": nbytes / t / 1e9, "frac": nbytes / t / 1e9 / pk["hbm_gbs"]}
    del qX
    # offline weight rotation of W_down (4096 x 16384 fp32, 268 MB in and out), random signs
    Wd = torch.from_numpy(W).to(dev)
    sg = torch.from_numpy(inputs.random_signs(K_IN)).to(dev)
    Wr = torch.empty_like(Wd)
    t = ev_time(lambda i: hbl.rotate_weights(Wd, sg, out=Wr), 1, 10)
    nbytes = 2 * N_OUT * K_IN * 4
    others["rotate_weights"] = {"workload": "W_down 4096 x 16384 fp32, random signs",
                                "us": t * 1e6, "bytes": nbytes, "achieved_gbs": nbytes / t / 1e9,
                                "frac": nbytes / t / 1e9 / pk["hbm_gbs"]}
    del Wd, Wr
    # QKV / KV-cache quantiser: 8192 tokens x 96 heads x 128 (201 MB bf16)
    QX = torch.from_numpy(inputs.qkv_states().view(np.int16)).view(torch.bfloat16).to(dev)
    rows = QX.numel() // 128
    ksc = torch.empty(rows, dtype=torch.float32, device=dev)
    for kb in (3, 4, 8):
        kc = torch.empty((rows, 128 * kb // 8), dtype=torch.uint8, device=dev)
        t = ev_time(lambda i: hbl.kv_quant(QX, kb, out=(kc, ksc)), 1, 20)
        nbytes = rows * 128 * 2 + rows * 128 * kb // 8 + rows * 4
        others["kv_quant_%dbit" % kb] = {
            "workload": "qkv 8192 x 96 x 128 after RoPE", "us": t * 1e6, "bytes": nbytes,
            "achieved_gbs": nbytes / t / 1e9, "frac": nbytes / t / 1e9 / pk["hbm_gbs"]}
        del kc
    del QX
    clocks = sampler.stop()

    # ---- end to end through the host-buffer call: H2D X, forward, D2H Y
    Xh = torch.from_numpy(X_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M_TOK, N_OUT), dtype=torch.bfloat16).pin_memory()
    hws = torch.empty(hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD_HOSTIO, M_TOK, K_IN, N_OUT,
                                         BITS), dtype=torch.uint8, device=dev)
    del Xd
    for _ in range(2):
        hbl.hbitlinear_forward_hostio(Xh, packed, alpha, BITS, Yh, hws, status=status)
    barrier()
    e2e_steps = max(3, min(args.steps, 20))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        hbl.hbitlinear_forward_hostio(Xh, packed, alpha, BITS, Yh, hws, status=status)
    b.record(stream)
    barrier()
    t_e2e = hdist.max_over_ranks(a.elapsed_time(b), dev) * 1e-3
    e2e_value = world * M_TOK * e2e_steps / t_e2e
    st = int(status[0].item())

    # ---- roofline of the dominant kernel
    ops = 2.0 * M_TOK * N_OUT * K_IN
    if t_k2 >= t_k1:
        achieved = ops / t_k2 / 1e12
        # the GEMM is timed in a sub-second loop at full clocks: the burst rate
        # of the same MMA instruction measured by the probe on this GPU
        peak = int8_probe["tops"]
        roof = {"bound": "tensor",
                "kernel": "gemm_pair (TMA-fed tcgen05.mma.cta_group::2 kind::i8 on pairs of SMs, "
                          "256 x 256 tiles, accumulators in TMEM)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_note": "dense INT8 (TOPS) measured on this GPU by hbl_probe_tc_int8: %d "
                             "SMs x %d back-to-back tcgen05.mma kind::i8 128x256x32 from shared "
                             "memory, best of 5, CUDA events; for context 2 x %s burst bf16 = "
                             "%.1f (frac %.2f) and the 4500 TOPS datasheet figure (frac %.2f)"
                             % (n_sms, int8_probe["mmas_per_cta"], pk["source"],
                                2.0 * pk["bf16_tflops"], achieved / (2.0 * pk["bf16_tflops"]),
                                achieved / 4500.0),
                "traffic": recorded_traffic("gemm_pair_a4_ffn_wdown",
                                            source_hash("k10_gemm_pair.cu")),
                "us_per_launch": t_k2 * 1e6}
    else:
        nbytes = M_TOK * K_IN * 2 + M_TOK * K_IN + 8 * M_TOK  # one-byte codes in the forward
        achieved = nbytes / t_k1 / 1e9
        roof = {"bound": "hbm", "kernel": "norm_fwht_quant", "achieved": achieved,
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                "traffic": recorded_traffic("norm_fwht_quant_a4_ffn_wdown",
                                            source_hash("k1_impl.cuh")),
                "us_per_launch": t_k1 * 1e6}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_TOK, "K": K_IN, "N": N_OUT, "act_bits": BITS,
                   "global_batch": world * M_TOK,
                   "parallelism": "replicas by token rows (no collective)" if world > 1
                   else "single GPU",
                   "l2": "inputs larger than L2 (X 268 MB per step)"},
        "roofline": roof,
        "kernels_us": {"norm_fwht_quant": t_k1 * 1e6, "expand_ternary": t_kx * 1e6,
                       "gemm_pair": t_k2 * 1e6},
        "kernels_note": "the stages as separate calls, timed one after another; the forward "
                        "runs two kernels: norm_fwht_quant widening the packed weights beside "
                        "its rows, then gemm_pair",
        "norm_fwht_quant_views": {
            "hbm": {"bytes": M_TOK * K_IN * 3 + 8 * M_TOK,
                    "achieved_gbs": (M_TOK * K_IN * 3 + 8 * M_TOK) / t_k1 / 1e9,
                    "frac": (M_TOK * K_IN * 3 + 8 * M_TOK) / t_k1 / 1e9 / pk["hbm_gbs"]},
            "alu": fp32_view(M_TOK * K_IN, 14, t_k1, n_sms, SM_MAX_MHZ)},
        "quant": quant,
        "decode": decode,
        "others": others,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": M_TOK * K_IN * 2,
                "d2h_bytes_per_step": M_TOK * N_OUT * 2, "steps": e2e_steps,
                "api": "hbl_hbitlinear_forward_hostio (pinned host buffers)"},
        # per forward at this shape: K1 (widening the weights beside its rows), the
        # GEMM (the ncu launch list of `--only forward`; the host plan check)
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "device_status": st,
        "peaks": dict(pk, int8_tops_probe=probe_tops),
        "int8_probe": int8_probe,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        wp, wa = oracle.pack_ternary(W)
        line["cpu_baseline"] = cpu_baseline(X_bits, wp, wa)
    if rank == 0:
        print(json.dumps(line))
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def run_only(args):
    """A single case with few launches, sized for profiler captures."""
    import numpy as np
    import torch

    import hadamard_rotated_int4_b200 as hbl
    from hadamard_rotated_int4_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.only.startswith("quant"):
        bits = int(args.only[-1])
        X = torch.from_numpy(inputs.activations("quant").view(np.int16)).view(
            torch.bfloat16).to(dev)
        fn = lambda: hbl.norm_fwht_quant(X, bits)
    elif args.only in ("nohad4", "ln4"):
        X = torch.from_numpy(inputs.activations("quant").view(np.int16)).view(
            torch.bfloat16).to(dev)
        fl = hbl.NORM_NO_HADAMARD if args.only == "nohad4" else hbl.NORM_LAYERNORM
        fn = lambda: hbl.norm_quant(X, 4, fl)
    elif args.only == "rotate":
        Wd = torch.from_numpy(inputs.weights("ffn_wdown")).to(dev)
        sg = torch.from_numpy(inputs.random_signs(K_IN)).to(dev)
        Wr = torch.empty_like(Wd)
        fn = lambda: hbl.rotate_weights(Wd, sg, out=Wr)
    elif args.only.startswith("kv"):
        QX = torch.from_numpy(inputs.qkv_states().view(np.int16)).view(torch.bfloat16).to(dev)
        kb = int(args.only[2:])
        fn = lambda: hbl.kv_quant(QX, kb)
    elif args.only.startswith("decode"):  # 1 (or 32) tokens through W_o or W_down
        Kd = 4096 if args.only.startswith("decode_wo") else 16384
        T = 32 if args.only.endswith("_t32") else 1
        name = "decode_wo" if Kd == 4096 else "decode_wdown"
        Xt = torch.from_numpy(inputs.activations(name, M=T, K=Kd, seed=1).view(
            np.int16)).view(torch.bfloat16).to(dev)
        pd, ad = hbl.pack_ternary(torch.from_numpy(inputs.latent_weights(N_OUT, Kd, seed=7)).to(dev))
        wsd = torch.empty(max(16, hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, T, Kd, N_OUT,
                                                     BITS)), dtype=torch.uint8, device=dev)
        fn = lambda: hbl.hbitlinear_forward(Xt, pd, ad, BITS, ws=wsd)
    elif args.only in ("gemv_rows", "gemv_splitk"):
        # the CUDA-core GEMVs: one weight row per warp (4 tokens, K = 16384),
        # split-K with a reduction kernel (8 tokens, K = 1024); N = 4096
        Kd = 16384 if args.only == "gemv_rows" else 1024
        Mt = 4 if args.only == "gemv_rows" else 8
        Xt = torch.from_numpy(inputs.activations("decode_wdown", M=Mt, K=Kd, seed=1).view(
            np.int16)).view(torch.bfloat16).to(dev)
        pd, ad = hbl.pack_ternary(torch.from_numpy(inputs.latent_weights(N_OUT, Kd, seed=7)).to(dev))
        codes, scales, rowsum = hbl.norm_fwht_quant(Xt, BITS)
        fn = lambda: hbl.ternary_gemm(codes, scales, rowsum, BITS, Kd, pd, ad, path=hbl.PATH_GEMV)
    elif args.only in ("pack", "expand"):
        Wd = torch.from_numpy(inputs.weights("ffn_wdown")).to(dev)
        pd, ad = hbl.pack_ternary(Wd)
        if args.only == "pack":
            fn = lambda: hbl.pack_ternary(Wd)
        else:
            del Wd
            Ws = torch.empty((N_OUT, K_IN), dtype=torch.int8, device=dev)
            fn = lambda: hbl.expand_ternary(pd, K_IN, out=Ws)
    elif args.only == "int8_probe":
        st = hbl.new_status(dev)
        n = torch.cuda.get_device_properties(dev).multi_processor_count
        fn = lambda: hbl.probe_tc_int8(n, 1 << 12, st)
    else:
        X = torch.from_numpy(inputs.activations("ffn_wdown").view(np.int16)).view(
            torch.bfloat16).to(dev)
        packed, alpha = hbl.pack_ternary(torch.from_numpy(inputs.weights("ffn_wdown")).to(dev))
        if args.only == "forward":
            ws = torch.empty(hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, M_TOK, K_IN, N_OUT,
                                                BITS), dtype=torch.uint8, device=dev)
            fn = lambda: hbl.hbitlinear_forward(X, packed, alpha, BITS, ws=ws)
        elif args.only == "gemm_packed":  # the tensor-core GEMM on the packed weights
            B8 = hbl.ACT_INT4_BYTES
            codes, scales, rowsum = hbl.norm_fwht_quant(X, B8)
            Yp = torch.empty((M_TOK, N_OUT), dtype=torch.bfloat16, device=dev)
            fn = lambda: hbl.ternary_gemm(codes, scales, rowsum, B8, K_IN, packed, alpha, out=Yp,
                                          path=hbl.PATH_TC_PACKED)
        elif args.only == "gemm_pair":  # the paired-SM GEMM (weights expanded by the call)
            B8 = hbl.ACT_INT4_BYTES
            codes, scales, rowsum = hbl.norm_fwht_quant(X, B8)
            Yp = torch.empty((M_TOK, N_OUT), dtype=torch.bfloat16, device=dev)
            fn = lambda: hbl.ternary_gemm(codes, scales, rowsum, B8, K_IN, packed, alpha, out=Yp,
                                          path=hbl.PATH_TC_PAIR)
        else:  # the forward's GEMM: one-byte INT4 codes, expanded weights
            B8 = hbl.ACT_INT4_BYTES
            codes, scales, rowsum = hbl.norm_fwht_quant(X, B8)
            Ws = hbl.expand_ternary(packed, K_IN)
            fn = lambda: hbl.ternary_gemm_s8w(codes, scales, B8, Ws, alpha)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"only": args.only, "steps": args.steps,
                      "us_per_step": 1e3 * a.elapsed_time(b) / max(1, args.steps)}))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_only(args)
    return run_hbl(args)


if __name__ == "__main__":
    sys.exit(main())
