"""Register and spill budgets of the kernels, from ptxas's resource report (CPU only).

The occupancy the kernels are designed for depends on these numbers:

* the token-block quantizer must fit in 64 registers, so that 4 CTAs of 256
  threads (or 2 of 512) share an SM's 65,536 registers;
* the channel-mean kernels must not spill;
* the attention kernel runs 384 threads per CTA, one CTA per SM, and its
  setmaxnreg split assumes a launch of at most 168 registers per thread
  (384 x 168 = 64,512). Its spills must stay a few bytes.

nvcc compiles for sm_100a without a GPU. Only ptxas's printed summary
(`-Xptxas -v`) is read.
"""

import os
import re
import subprocess

import pytest

from precision_attention_fmha_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "precision_attention_fmha_b200", "csrc")


def resources(src, tmp_path):
    cmd = [build_mod.nvcc()] + build_mod.ARCH + [f for f in build_mod.FLAGS] + [
        "-c", os.path.join(CSRC, src), "-o", str(tmp_path / (src + ".o"))]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    out = {}
    name = None
    for line in (r.stdout + r.stderr).splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            name = m.group(1)
            out[name] = {"regs": None, "spill_st": 0, "spill_ld": 0}
            continue
        if name is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            out[name]["spill_st"], out[name]["spill_ld"] = int(m.group(1)), int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            out[name]["regs"] = int(m.group(1))
    return out


@pytest.fixture(scope="module")
def quant_res(tmp_path_factory):
    return resources("quantize.cu", tmp_path_factory.mktemp("ptxas"))


def test_token_block_quantizer_fits_its_occupancy(quant_res):
    """Without a shift: 4 CTAs of 256 or 2 of 512 per SM (64 registers a thread);
    with one: 3 CTAs of 256 (85 registers) or 1 of 512."""
    tb = {}
    for n, r in quant_res.items():
        m = re.search(r"quant_token_block_kernelILb[01]ELi(256|512)ELb([01])E", n)
        if m:
            tb[n] = (int(m.group(1)), m.group(2) == "1", r)
    assert len(tb) == 8, sorted(quant_res)  # INT8 and E4M3, two CTA sizes, with and without a shift
    for n, (threads, shift, r) in tb.items():
        limit = (85 if threads == 256 else 128) if shift else 64
        assert r["regs"] is not None and r["regs"] <= limit, (n, r)
        assert r["spill_st"] == 0 and r["spill_ld"] == 0, (n, r)


def test_quantizer_and_mean_kernels_do_not_spill(quant_res):
    assert any("channel_mean_partial_kernel" in n for n in quant_res)
    assert any("channel_mean_final_kernel" in n for n in quant_res)
    for n, r in quant_res.items():
        assert r["spill_st"] == 0 and r["spill_ld"] == 0, (n, r)


# The D = 192 kernel with BF16 Q/K and E4M3 V (one query tile, two softmax
# warpgroups splitting its KV tiles, a second producer warp for the V ring)
# spills a few registers in its softmax region (12 bytes stored, about 560
# bytes of reloads). Measured on a B200 it is still the faster build: 61.3 %
# of its peak against 53.9 % for the one-producer build that does not spill.
SPILL_ALLOWED = {"AttnCfgILi192ELi0ELi1E": 640}


@pytest.mark.parametrize("src,min_kernels", [("attn_pv8.cu", 4), ("attn_d192.cu", 6)])
def test_attention_kernel_register_budget(tmp_path, src, min_kernels):
    res = resources(src, tmp_path)
    attn = {n: r for n, r in res.items() if "attn_fwd_kernel" in n}
    assert len(attn) >= min_kernels
    for n, r in attn.items():
        limit = next((v for k, v in SPILL_ALLOWED.items() if k in n), 64)
        assert r["regs"] is not None and r["regs"] <= 168, (n, r)
        assert r["spill_st"] <= 64 and r["spill_ld"] <= limit, (n, r)
