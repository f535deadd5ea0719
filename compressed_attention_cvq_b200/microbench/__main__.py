"""Run the unit-throughput probes on GPU 0 and print one JSON object.

    python -m compressed_attention_cvq_b200.microbench [kind ...]   # all probes, or only these

Builds microbench/libcvq_micro.so on first use (nvcc, sm_100a).  For each probe:
operations per second and per SM per clock at the median SM clock sampled while it
ran (nvidia-smi) and at the 1965 MHz maximum.
"""
import ctypes
import json
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libcvq_micro.so")
KINDS = {0: "ffma", 1: "ffma2 (f32x2, 2 FMA each)", 2: "sincos (__sincosf)", 3: "exp2",
         4: "lds128 conflict-free", 5: "lds128 random", 6: "atomicAdd f32 distinct banks",
         7: "atomicAdd f32 random", 8: "atomicAdd f32 same address", 9: "shfl_xor",
         10: "red.shared.add.f32 distinct", 11: "red.shared.add.u32 distinct",
         12: "red.shared.add.u64 distinct", 13: "plain f32 ld/add/st distinct",
         14: "plain float4 ld/add/st conflict-free", 15: "mixed: lds128 + 2 x red.f32",
         16: "red.global.add.v4.f32 random (L2, 64 KB per CTA)",
         17: "red.global.add.f32 random (L2, 64 KB per CTA)",
         18: "red.global.add.v4.f32, 25% on 4 hot slots",
         19: "red.shared::cluster.add.f32 distinct (own CTA)",
         20: "warp-owned float4 bins, ld/add/st, equal codes take turns (uniform codes)",
         21: "warp-owned float4 bins, ld/add/st, equal codes take turns (25% code 0)"}
ITERS = {0: 4000, 1: 2000, 2: 1000, 3: 1000, 4: 4000, 5: 4000, 6: 2000, 7: 2000, 8: 500, 9: 2000, 10: 2000, 11: 2000, 12: 2000, 13: 2000, 14: 2000, 15: 2000,
         16: 200, 17: 200, 18: 100, 19: 2000, 20: 500, 21: 500}
GLOBAL_KINDS = (16, 17, 18)     # take a scratch buffer of blocks x 16384 floats


def build():
    sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
    from compressed_attention_cvq_b200.build import ARCH, nvcc
    src = os.path.join(HERE, "microbench.cu")
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(src):
        subprocess.check_call([nvcc(), *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                               "-shared", "-cudart", "static", src, "-o", LIB])
    lib = ctypes.CDLL(LIB)
    lib.cvqmb_run.restype = ctypes.c_double
    lib.cvqmb_run.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_void_p, ctypes.c_void_p]
    return lib


def main():
    import torch
    lib = build()
    dev = torch.device("cuda", 0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    out = torch.zeros(4096, device=dev)
    stream = torch.cuda.current_stream()
    res = {"sm_count": sms}
    smi = subprocess.Popen(["nvidia-smi", "-i", "0", "--query-gpu=clocks.sm",
                            "--format=csv,noheader,nounits", "-lms", "100"],
                           stdout=subprocess.PIPE, text=True)
    rows = {}
    scratch = None
    only = [int(k) for k in sys.argv[1:]]
    for kind, name in KINDS.items():
        if only and kind not in only:
            continue
        blocks, threads = sms * 4, 256
        dst = out
        if kind in GLOBAL_KINDS:
            if scratch is None:
                scratch = torch.zeros(blocks * 16384, device=dev)
            dst = scratch
        for _ in range(2):
            lib.cvqmb_run(kind, blocks, threads, ITERS[kind] // 10, ctypes.c_void_p(dst.data_ptr()),
                          ctypes.c_void_p(stream.cuda_stream))
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ops = lib.cvqmb_run(kind, blocks, threads, ITERS[kind], ctypes.c_void_p(dst.data_ptr()),
                            ctypes.c_void_p(stream.cuda_stream))
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        rows[name] = {"ops": ops, "ms": ms, "ops_per_s": ops / (ms * 1e-3)}
    smi.terminate()
    clocks = [float(x) for x in smi.stdout.read().split() if x.strip().replace(".", "").isdigit()]
    busy = [c for c in clocks if c > 500] or [1965.0]
    busy.sort()
    f = busy[len(busy) // 2]
    for name, r in rows.items():
        r["per_sm_per_clk_at_sampled"] = r["ops_per_s"] / (sms * f * 1e6)
        r["per_sm_per_clk_at_1965"] = r["ops_per_s"] / (sms * 1965e6)
    res["sm_mhz_median"] = f
    res["probes"] = rows
    print(json.dumps(res, indent=1))


if __name__ == "__main__":
    main()
