"""Helpers shared by the GPU parity tests: move a seeded workload to the device, run
the library on it, and run the float64 oracle on the same inputs."""
import numpy as np
import torch

from oracle import cvq_oracle as O

OUT_TOL = 2e-3        # max |out - oracle|
LSE_RTOL = 1e-4       # |lse - oracle| / max(|oracle|, 1)


def to_device(d, dev="cuda"):
    if d["q_dtype"] == "bf16":
        q = torch.from_numpy(d["q_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        q = torch.from_numpy(d["q"]).to(dev)
    return dict(q=q,
                key_cb=torch.from_numpy(d["key_cb"]).to(dev),
                val_cb=torch.from_numpy(d["val_cb"]).to(dev),
                key_codes=torch.from_numpy(d["key_codes"]).to(dev),
                val_codes=torch.from_numpy(d["val_codes"]).to(dev),
                seq_lens=torch.from_numpy(d["seq_lens"]).to(dev))


def run_gpu(d, form="gqa", n_splits=None, dd=None):
    import compressed_attention_cvq_b200 as cvq
    dd = dd or to_device(d)
    out, lse = cvq.attend(dd["q"], dd["key_cb"], dd["val_cb"], dd["key_codes"], dd["val_codes"],
                          dd["seq_lens"], rope_base=d["rope_base"], n_splits=n_splits, form=form)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def run_oracle(d, heads=None):
    return O.attend(d["q"], d["key_cb"], d["val_cb"], d["key_codes"], d["val_codes"],
                    d["seq_lens"], d["rope_base"], heads=heads,
                    codes_layout=d.get("codes_layout", "token"))


def assert_close(out, lse, ref_out, ref_lse, heads=None, out_tol=OUT_TOL, lse_rtol=LSE_RTOL):
    if heads is None:
        B, Hq = ref_lse.shape
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    worst_o, worst_l = 0.0, 0.0
    for b, h in heads:
        if np.isneginf(ref_lse[b, h]):
            assert np.isneginf(lse[b, h]), (b, h, lse[b, h])
            assert np.all(out[b, h] == 0), (b, h)
            continue
        eo = float(np.max(np.abs(out[b, h] - ref_out[b, h])))
        el = abs(lse[b, h] - ref_lse[b, h]) / max(abs(ref_lse[b, h]), 1.0)
        worst_o, worst_l = max(worst_o, eo), max(worst_l, el)
    assert worst_o <= out_tol, f"max |out - oracle| = {worst_o:.3e} > {out_tol}"
    assert worst_l <= lse_rtol, f"lse rel err = {worst_l:.3e} > {lse_rtol}"
    return worst_o, worst_l
