"""Static checks on the CUDA sources (no GPU).

Warp-synchronous instructions -- the `.sync.aligned` tcgen05 loads, stores and
waits, TMEM allocation, `setmaxnreg`, and warp votes and shuffles -- must be
executed by all 32 lanes of a warp together; run by part of a warp they are
undefined and can stall it where no bounded wait can see.  Branches on a
per-row value (the row's allowed-key limit in a tile, whether the row exists,
whether the row moved its softmax reference) diverge within a warp, so none of
those instructions may appear inside one.
"""
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "video_diffusion_transformer_attention_b200", "csrc")
KERNELS = ["attn_fwd_sm100.cuh", "attn_cross_sm100.cuh", "attn_cross_fp8_sm100.cuh", "attn_fwd_fp8_sm100.cuh", "fp8_quant.cuh",
           "qk_norm.cuh", "attn_merge.cuh", "vsmooth_group.cuh"]
PTX_HELPERS = ["sm100_ptx.cuh", "sm100_fp8_ptx.cuh"]
WARP_INTRINSICS = {"__syncwarp", "__any_sync", "__all_sync", "__ballot_sync", "__shfl_sync",
                   "__shfl_xor_sync", "__shfl_down_sync", "__match_any_sync"}
# conditions on per-row values used by the kernels
PER_ROW_IF = re.compile(r"\bif \((lim < kBlockN|row < p\.Sq|rescale|p\.lse != nullptr && row < p\.Sq)\)")


def _block(src, open_idx):
    """Text between the brace at open_idx and its match."""
    depth = 0
    for i in range(open_idx, len(src)):
        if src[i] == "{":
            depth += 1
        elif src[i] == "}":
            depth -= 1
            if depth == 0:
                return src[open_idx + 1:i]
    raise ValueError("unbalanced braces")


def _strip_comments(src):
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def warp_synchronous_helpers():
    """Device helpers whose body issues a .sync.aligned instruction, plus the warp intrinsics."""
    names = set(WARP_INTRINSICS)
    for f in PTX_HELPERS:
        src = open(os.path.join(CSRC, f)).read()
        for m in re.finditer(r"__device__ __forceinline__ [^;{]*?\b(\w+)\s*\([^;{]*\)\s*\{", src):
            if ".sync.aligned" in _block(src, m.end() - 1):
                names.add(m.group(1))
    # kernel-level helpers built on them
    names.add("warp_wait")
    return names


def per_row_violations(src, helpers):
    """(condition, helper) pairs where a per-row branch body calls a warp-synchronous helper."""
    src = _strip_comments(src)
    found = []
    for m in PER_ROW_IF.finditer(src):
        rest = src[m.end():]
        stripped = rest.lstrip()
        if stripped.startswith("{"):
            body = _block(src, m.end() + (len(rest) - len(stripped)))
        else:
            body = stripped.split(";", 1)[0]
        for name in helpers:
            if re.search(r"\b" + re.escape(name) + r"\s*[(<]", body):
                found.append((m.group(1), name))
    return found


def test_helper_scan_finds_the_tmem_and_register_split_helpers():
    helpers = warp_synchronous_helpers()
    for name in ("tmem_ld32", "tmem_ld_wait", "tmem_st16", "tmem_st32", "tmem_st_wait", "tmem_alloc",
                 "setmaxnreg_inc", "setmaxnreg_dec"):
        assert name in helpers, name


def test_checker_flags_a_wait_inside_a_per_row_branch():
    helpers = warp_synchronous_helpers()
    planted = """
        if (lim < kBlockN) {
            tmem_ld_wait(s[2]);
            for (int i = 0; i < 32; ++i) s[0][i] = 0;
        }
    """
    assert per_row_violations(planted, helpers) == [("lim < kBlockN", "tmem_ld_wait")]
    assert per_row_violations("if (rescale) __syncwarp();", helpers) == [("rescale", "__syncwarp")]
    clean = "if (row < p.Sq) { dst[0] = v; }  if (__any_sync(0xffffffffu, rescale)) { tmem_ld32(a, o); }"
    assert per_row_violations(clean, helpers) == []


@pytest.mark.parametrize("name", KERNELS)
def test_no_warp_synchronous_instruction_in_a_per_row_branch(name):
    src = open(os.path.join(CSRC, name)).read()
    assert per_row_violations(src, warp_synchronous_helpers()) == []
