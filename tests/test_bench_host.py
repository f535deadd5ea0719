"""Host-side checks of bench.py's accounting (no GPU): the algorithmic FLOPs and bytes per
layer step, the shared-memory floor, the append work and the whole-job rate, each against a
value worked out by hand from the definitions in the docstrings (per token and query head:
64 pairs x (2 mul + 2 add) = 256 FLOP, + 128 (R - 1) to sum rounds, + one bin add per
(group, round); per token and KV head: one code byte per (group, round) for keys and for
values)."""
import math
import os

import pytest

import bench
import workloads

W = workloads.WORKLOADS


def test_algorithmic_flops_by_hand():
    # 128K layer, R = 1: 131072 tokens x 32 heads x (256 + 0 + 16)
    assert bench.algorithmic_flops(W["llama8b_layer_T131072_R1"], 131072) == 131072 * 32 * 272
    # 32K layer, R = 2: 256 + 128 + 32 = 416 per token and head
    assert bench.algorithmic_flops(W["llama8b_layer_T32768_R2"], 32768) == 32768 * 32 * 416
    # paper's 1-bit setting, R = 11 over 2 groups: 256 + 1280 + 22 = 1558
    assert bench.algorithmic_flops(W["llama8b_layer_T131072_R11_g64"], 131072) == 131072 * 32 * 1558


def test_code_bytes_by_hand():
    # 128K layer, R = 1: codes 131072 x 8 KV heads x (16 key + 16 value bytes) = 33,554,432;
    # codebooks 2 x 8 heads x 16 groups x 256 codewords x 8 floats x 4 B = 2,097,152
    assert bench.code_bytes(W["llama8b_layer_T131072_R1"], 131072) == 33_554_432 + 2_097_152
    # R = 11 over 64-scalar groups: codes 131072 x 8 x 2 x 2 x 11; codebooks
    # 2 x 8 x 2 groups x 11 rounds x 64 codewords x 64 floats x 4 B
    assert bench.code_bytes(W["llama8b_layer_T131072_R11_g64"], 131072) == (
        131072 * 8 * 2 * 2 * 11 + 2 * 8 * 2 * 11 * 64 * 64 * 4)


def test_smem_floor_by_hand():
    # per token and KV head at R = 1: 512 B of codewords at 125.6 B/clk and 16 groups x 4
    # heads of bin atomics at 7.73 lanes/clk, over 148 SMs at 1965 MHz
    clk = 512 / 125.6 + 64 / 7.73
    expect = 131072 * 8 * clk / 148 / 1965
    got = bench.smem_floor_us(W["llama8b_layer_T131072_R1"], 131072, 1965.0)
    assert math.isclose(got, expect, rel_tol=1e-12)
    assert 44.0 < got < 45.0


def test_encode_work_by_hand():
    # one append on the 128K layer (B = 1, 8 KV heads, R = 1): key and value, 16 groups x
    # 256 codewords x 8 dims x 3 FLOP each; bytes = both codebooks + the new vectors + codes
    flops, bytes_ = bench.encode_work(W["llama8b_layer_T131072_R1"])
    assert flops == 8 * 2 * 16 * 256 * 8 * 3
    assert bytes_ == 2 * 8 * 16 * 256 * 8 * 4 + 8 * (2 * 128 * 4 + 2 * 16)
    # 64-scalar groups, R = 11: 2 groups x 64 codewords x 64 dims per round
    flops, bytes_ = bench.encode_work(W["llama8b_layer_T131072_R11_g64"])
    assert flops == 8 * 2 * 11 * 2 * 64 * 64 * 3
    assert bytes_ == 2 * 8 * 11 * 2 * 64 * 64 * 4 + 8 * (2 * 128 * 4 + 2 * 2 * 11)


@pytest.mark.parametrize("world,units,ms,expect", [(1, 131072, 0.15, 131072 / 0.15e-3),
                                                   (4, 1000, 2.0, 4 * 1000 / 2e-3)])
def test_whole_job_rate(world, units, ms, expect):
    assert math.isclose(bench.whole_job_rate(world, units, ms), expect, rel_tol=1e-12)


def test_roofline_legs_by_hand():
    # 128K layer, R = 1, 1965 MHz, 148 SMs:
    #   FP32: 131072 x 32 x 272 FLOP / 2 = 570,425,344 FMA at 123.74 lanes/clk
    #         -> 4,609,870.2 clk per SM-set -> / (148 x 1.965e9) = 15.851 us
    #   SFU:  131072 x 64 sin+cos pairs at 7.95 + 131072 x 32 exp2 at 15.90 per clk
    #         -> 1,055,173.0 + 263,791.1 = 1,318,964.2 clk -> 4.5353 us
    #   HBM:  35,651,584 B at 6528.7 GB/s -> 5.4607 us
    legs = bench.roofline_legs(W["llama8b_layer_T131072_R1"], 131072, 1965.0, 6528.7)
    clk = 148 * 1965e6
    assert math.isclose(legs["fp32_us"], 570_425_344 / 123.74 / clk * 1e6, rel_tol=1e-12)
    assert math.isclose(legs["fp32_us"], 15.851, rel_tol=1e-4)
    assert math.isclose(legs["sfu_us"], 4.5353, rel_tol=1e-4)
    assert math.isclose(legs["hbm_us"], 35_651_584 / 6528.7e9 * 1e6, rel_tol=1e-12)
    assert max(legs, key=legs.get) == "fp32_us"


def test_packed_code_bytes_by_hand():
    # the paper's 1-bit setting at 128K tokens: 131072 tokens x 8 KV heads x (key + value)
    # x 2 groups x 11 rounds = 46,137,344 codes; packed at 6 bits: 34,603,008 bytes (3/4)
    w = W["llama8b_layer_T131072_R11_g64"]
    cbs = 2 * 8 * 2 * 11 * 64 * 64 * 4
    assert bench.code_bytes(w, 131072, 6) == 34_603_008 + cbs
    assert bench.code_bytes(w, 131072, 8) == 46_137_344 + cbs
    class A:  # noqa: E701 - stand-in for the parsed arguments
        code_bits = 0
    assert bench.code_bits_of(w, A) == 6 and bench.code_bits_of(W["llama8b_layer_T131072_R1"], A) == 8


def _unresolved_globals(path):
    """Names that a function of the file reads as globals but that neither the module
    defines (assignment, import, def, class) nor Python provides (builtins)."""
    import builtins
    import symtable

    src = open(path).read()
    top = symtable.symtable(src, path, "exec")
    defined = {s.get_name() for s in top.get_symbols()
               if s.is_assigned() or s.is_imported() or s.is_namespace()}
    known = defined | set(dir(builtins)) | {"__file__", "__name__"}
    bad = []

    def walk(t):
        for ch in t.get_children():
            for s in ch.get_symbols():
                if s.is_referenced() and s.is_global() and s.get_name() not in known:
                    bad.append(f"{ch.get_name()}: {s.get_name()}")
            walk(ch)

    walk(top)
    return bad


def _python_sources():
    import glob

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = []
    for sub in ("*.py", "compressed_attention_cvq_b200/**/*.py", "oracle/*.py", "tests/**/*.py"):
        out += [os.path.relpath(p, root) for p in glob.glob(os.path.join(root, sub), recursive=True)]
    return sorted(out)


@pytest.mark.parametrize("rel", _python_sources())
def test_every_global_name_resolves(rel):
    """A function that reads a name its module never binds (a missing import) fails only
    when that function runs, on a GPU machine for most of these files: check statically."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    assert _unresolved_globals(os.path.join(root, rel)) == []
