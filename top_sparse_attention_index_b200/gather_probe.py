"""The gather-rate probe, run from Python: the SM-side roofline of the sparse-attention
gather on the device at hand.

The fused kernel's K/V rows are gathered at random from a cache that, at the long-prefill
shape (article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in CANN
prefill PR", section "Nine tests that passed, and a speed number that did not come from
this branch"), is about the size of B200's L2, so nearly every gathered row is an L2 hit
and HBM bandwidth is not the bound.  The probe kernel (include/qsa_probe.h) does the
kernel's data movement without its arithmetic: random rows of an L2-resident buffer into
shared memory, each landed row read back once with ldmatrix.  gather_peak() runs it over
the loaders (the kernel's cp.async, and TMA tile::gather4) and a few pipeline shapes and
returns the best rate; the benchmark reports the fused kernel against it.

    python -m top_sparse_attention_index_b200.gather_probe [--rows 512|256] [--sweep] [--mma]

prints one JSON line per run (--sweep: every method, with and without the read-back,
over more shapes; --mma: the shared-memory operand rates of ldmatrix and tcgen05.mma,
mma_operand_rates()).  Needs a GPU; allocates a 64 MB buffer.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

# The gather probe (include/qsa_probe.h) measures, live on the device, the rate at which
# the SMs pull random rows of an L2-resident 64 MB buffer into shared memory and read each
# landed row back once with ldmatrix -- the data movement of the fused kernel without its
# arithmetic -- with the fused kernel's own loader (cp.async, method 0) and with TMA
# tile::gather4 (method 1), over a few pipeline shapes (warps per CTA, stages, CTAs per
# SM).  The best rate is the SM-side roofline of a launch whose gathered rows are L2 hits.
PROBE_BUFFER_BYTES = 64 << 20
PROBE_CONFIGS = {
    512: [(12, 2, 1), (8, 3, 1), (6, 2, 2), (2, 4, 3)],
    256: [(15, 3, 1), (12, 4, 1), (4, 4, 3), (4, 2, 3)],
}


def gather_peak(device, row_bytes: int, reps: int = 5) -> dict:
    """Best gather rate (TB/s) of the probe over its methods and pipeline shapes."""
    from . import _binding as qsa
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    gen = torch.Generator(device=device).manual_seed(99)
    buf = torch.randint(-2**31, 2**31 - 1, (PROBE_BUFFER_BYTES // 4,), dtype=torch.int32,
                        device=device, generator=gen)
    sink = torch.zeros(258, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    rows = PROBE_BUFFER_BYTES // row_bytes
    runs = []
    for method in (0, 1):
        for warps, stages, per_sm in PROBE_CONFIGS[row_bytes]:
            ctas = sms * per_sm
            iters = max(4, int(2e9 / (ctas * warps * 16 * row_bytes)))
            moved = ctas * warps * iters * 16 * row_bytes
            sink.zero_()

            def launch(seed):
                st = qsa.qsa_probe_gather(method, 1, buf.data_ptr(), rows, row_bytes, row_bytes,
                                          warps, stages, ctas, iters, seed, sink.data_ptr(),
                                          stream.cuda_stream)
                if st != qsa.QSA_OK:
                    raise qsa.QSAError(st, qsa.qsa_last_error_detail())

            launch(1)
            launch(2)
            times = []
            for r in range(reps):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                launch(3 + r)
                b.record(stream)
                torch.cuda.synchronize(device)
                times.append(a.elapsed_time(b) * 1e-3)
            ok = int(sink[0].item()) == 0
            runs.append({"method": ["cp.async", "tma gather4"][method], "warps_per_cta": warps,
                         "stages": stages, "ctas_per_sm": per_sm,
                         "tb_per_s": moved / statistics.median(times) / 1e12 if ok else None})
    best = max((r for r in runs if r["tb_per_s"] is not None), key=lambda r: r["tb_per_s"])
    return {"tb_per_s": best["tb_per_s"], "best": best, "runs": runs, "row_bytes": row_bytes,
            "buffer_bytes": PROBE_BUFFER_BYTES, "read_back": True}


SWEEP_CONFIGS = {
    512: [(12, 2, 1), (8, 3, 1), (6, 4, 1), (4, 2, 3), (4, 3, 2), (6, 2, 2), (2, 4, 3), (8, 2, 1)],
    256: [(12, 4, 1), (15, 3, 1), (8, 4, 1), (4, 4, 3), (4, 3, 3), (6, 4, 2), (2, 4, 3), (4, 2, 3)],
}


def sweep(device, row_bytes: int, reps: int = 5):
    """Every method (0: cp.async, 1: TMA gather4 from one lane per warp, 2: from one
    producer warp, 3: from several lanes of each warp) with and without the read-back,
    over SWEEP_CONFIGS; also checks the shared-memory layout of every method once
    (read_back 2).  Yields one dict per run."""
    from . import _binding as qsa
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    gen = torch.Generator(device=device).manual_seed(99)
    buf = torch.randint(-2**31, 2**31 - 1, (PROBE_BUFFER_BYTES // 4,), dtype=torch.int32,
                        device=device, generator=gen)
    sink = torch.zeros(258, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    rows = PROBE_BUFFER_BYTES // row_bytes
    plan = [(m, 2, (4, 2, 1)) for m in range(4)]
    plan += [(m, rb, c) for m in range(4) for rb in (0, 1) for c in SWEEP_CONFIGS[row_bytes]]
    for method, read_back, (warps, stages, per_sm) in plan:
        if method == 2 and warps + 1 > 16:
            continue
        ctas = sms * per_sm
        iters = max(4, int((0.2e9 if read_back == 2 else 2e9) / (ctas * warps * 16 * row_bytes)))
        moved = ctas * warps * iters * 16 * row_bytes
        sink.zero_()
        times = []
        for r in range(reps + 2):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            st = qsa.qsa_probe_gather(method, read_back, buf.data_ptr(), rows, row_bytes,
                                      row_bytes, warps, stages, ctas, iters, 1 + r,
                                      sink.data_ptr(), stream.cuda_stream)
            b.record(stream)
            if st != qsa.QSA_OK:
                raise qsa.QSAError(st, qsa.qsa_last_error_detail())
            torch.cuda.synchronize(device)
            if r >= 2:
                times.append(a.elapsed_time(b) * 1e-3)
        yield {"method": method, "read_back": read_back, "row_bytes": row_bytes,
               "warps_per_cta": warps, "stages": stages, "ctas_per_sm": per_sm,
               "tb_per_s": moved / statistics.median(times) / 1e12,
               "timeouts": int(sink[0].item()), "layout_mismatches": int(sink[1].item())}


MMA_N = (16, 32, 64, 128, 256)


def mma_operand_rates(device, rounds: int = 2000) -> dict:
    """Shared-memory operand bytes per clock per SM of the two MMA forms (the MMA probe of
    include/qsa_probe.h, one CTA per SM): ldmatrix.x4 from 16 warps, and tcgen05.mma with
    M = 128, K = 16 and N = 16 ... 256 (the accumulator checked exactly).  The gathered rows
    are read from shared memory once whichever form reads them, so the faster reader at
    this path's skinny shapes (many slots x 8-16 heads) is the one that can raise the
    fused kernel's bound."""
    from . import _binding as qsa
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    out = torch.zeros(2 + sms, dtype=torch.int64, device=device)
    stream = torch.cuda.current_stream(device)

    def run(method, n, bytes_per_cta):
        for r in (1, rounds):  # a warm-up launch, then the measured one
            out.zero_()
            st = qsa.qsa_probe_mma_operands(method, n, r, sms, out.data_ptr(), stream.cuda_stream)
            if st != qsa.QSA_OK:
                raise qsa.QSAError(st, qsa.qsa_last_error_detail())
        torch.cuda.synchronize(device)
        o = out.cpu()
        cycles = int(o[2:].max())
        return {"timeouts": int(o[0]), "mismatches": int(o[1]), "cycles": cycles,
                "bytes_per_clk_per_sm": bytes_per_cta(rounds) / cycles}

    res = {"rounds": rounds, "ctas": sms,
           "ldmatrix_x4_16_warps": run(0, 0, lambda r: r * 16 * 128 * 512), "tcgen05": {}}
    for n in MMA_N:
        d = run(1, n, lambda r, n=n: r * 16 * (128 + n) * 32)
        mmas = rounds * 16
        d.update({"M": 128, "N": n, "K": 16, "clk_per_mma": d["cycles"] / mmas,
                  "mac_per_clk_per_sm": mmas * 128 * n * 16 / d["cycles"]})
        res["tcgen05"][str(n)] = d
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, choices=[512, 256], default=512,
                    help="row bytes: 512 (bf16, head dim 256) or 256 (E4M3 codes)")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--mma", action="store_true",
                    help="the MMA operand-rate probe instead (ldmatrix vs tcgen05.mma)")
    args = ap.parse_args()
    device = torch.device("cuda", 0)
    if args.mma:
        print(json.dumps(mma_operand_rates(device)))
    elif args.sweep:
        for r in sweep(device, args.rows):
            print(json.dumps(r), flush=True)
    else:
        print(json.dumps(gather_peak(device, args.rows)))


if __name__ == "__main__":
    main()
