"""The C-ABI library loads on a machine without a GPU, exports every entry point
include/wq.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import build as wq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "wq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if wq_build.needs_build():
        wq_build.build()
    return wq.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), f"libwq.so does not export {n}"
        assert n in wq._SIGS, f"binding has no signature for {n}"
    assert set(wq._SIGS) == set(names)


def test_status_strings_and_version(lib):
    assert wq.wq_version() == 101
    for code, name in wq.STATUS.items():
        assert lib.wq_status_string(code).decode().startswith(name)


def test_workspace_bytes(lib):
    assert wq.wq_workspace_bytes(4288, 2048, 6144, 8) == 4288 * 2048 + 17152
    # int4 codes are kept one per byte in the fused linear's workspace
    assert wq.wq_workspace_bytes(4288, 2048, 6144, 4) == 4288 * 2048 + 17152
    assert wq.wq_workspace_bytes(1, 128, 16, 8) == 256 + 256
    assert wq.wq_workspace_bytes(64, 100, 256, 8) == 0      # K not a multiple of 128
    assert wq.wq_workspace_bytes(64, 256, 250, 8) == 0      # N not a multiple of 16
    assert wq.wq_workspace_bytes(64, 256, 256, 6) == 0      # bits


FAKE = 1 << 20          # a 16-byte aligned, never dereferenced address
MIS = FAKE + 8


def _linear(lib, **kw):
    a = dict(x=FAKE, M=64, K=256, N=256, cinv=FAKE, sid=FAKE, alpha=FAKE, beta=FAKE, S=3, T=1,
             step=0, qw=FAKE, s_w=FAKE, bias=FAKE, y=FAKE, ws=FAKE, ws_bytes=1 << 30, st=None)
    a.update(kw)
    return lib.wq_linear_w4a8(a["x"], a["M"], a["K"], a["N"], a["cinv"], a["sid"], a["alpha"],
                              a["beta"], a["S"], a["T"], a["step"], a["qw"], a["s_w"], a["bias"],
                              a["y"], a["ws"], a["ws_bytes"], a["st"])


@pytest.mark.parametrize("kw,code", [
    (dict(K=100), 2), (dict(K=0), 2), (dict(K=65536), 2), (dict(N=250), 2), (dict(N=0), 2),
    (dict(M=-1), 2), (dict(x=None), 1), (dict(qw=None), 1), (dict(alpha=None), 1),
    (dict(ws=None), 1), (dict(x=MIS), 3), (dict(y=MIS), 3), (dict(ws=FAKE + 16), 3),
    (dict(step=1), 4), (dict(step=-1), 4), (dict(S=0), 4), (dict(S=256), 4), (dict(T=0), 4),
    (dict(ws_bytes=100), 4),
])
def test_linear_rejects_bad_arguments_on_host(lib, kw, code):
    assert _linear(lib, **kw) == code


def test_other_entry_points_reject_on_host(lib):
    assert lib.wq_act_quant(FAKE, 8, 256, None, FAKE, FAKE, 3, 1, 0, 6, FAKE, FAKE, None) == 4
    assert lib.wq_act_quant(FAKE, 8, 200, None, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, None) == 2
    assert lib.wq_pack_int4(FAKE, None, 16, 96, FAKE, FAKE, None) == 2
    assert lib.wq_pack_int4(None, None, 16, 128, FAKE, FAKE, None) == 1
    assert lib.wq_debug_gemm_s32(FAKE, 8, FAKE, 16, 24, 128, FAKE, None, 0, None) == 2
    assert lib.wq_debug_gemm_s32(FAKE, 5, FAKE, 16, 32, 128, FAKE, None, 0, None) == 4
    assert lib.wq_debug_gemm_s32(FAKE, 8, FAKE, 16, 32, 128, None, None, 0, None) == 1
    # 16 tokens x 128 channels x K = 4096: K is split, so the scratch is required
    assert lib.wq_debug_gemm_s32(FAKE, 8, FAKE, 16, 128, 4096, FAKE, None, 0, None) == 1
    assert lib.wq_debug_gemm_s32(FAKE, 8, FAKE, 16, 128, 4096, FAKE, FAKE + 16, 1 << 20,
                                 None) == 3
    assert lib.wq_debug_gemm_s32(FAKE, 8, FAKE, 16, 128, 4096, FAKE, FAKE, 64, None) == 4
    assert lib.wq_gemm_w4ax(FAKE, FAKE, 4, 16, 128, 32, FAKE, None, 3, 2, 2, FAKE, FAKE, None,
                            FAKE, None) == 4
    assert lib.wq_channel_scale(None, 4, FAKE, 4, 128, FAKE, FAKE, None) == 1


def test_gemm_ws_scratch_rule_on_host(lib):
    """wq_gemm_w4ax_ws: the scratch is needed exactly when K is split (few tokens,
    few output tiles); a missing, misaligned or short one is refused before any
    launch, and a shape that does not split needs none."""
    lib.wq_gemm_scratch_bytes.restype = ctypes.c_size_t
    n = lib.wq_gemm_scratch_bytes(16, 4096, 128)
    assert n > 0
    assert lib.wq_gemm_scratch_bytes(8512, 4096, 16384) == 0
    assert lib.wq_gemm_scratch_bytes(16, 100, 128) == 0  # invalid K
    args = [FAKE, FAKE, 8, 16, 4096, 128, FAKE, None, 3, 1, 0, FAKE, FAKE, None, FAKE]
    ws = ctypes.c_size_t
    assert lib.wq_gemm_w4ax_ws(*args, None, ws(0), None) == 1
    assert lib.wq_gemm_w4ax_ws(*args, FAKE + 16, ws(n), None) == 3
    assert lib.wq_gemm_w4ax_ws(*args, FAKE, ws(n - 1), None) == 4
    # the usual checks first: a bad act_bits is refused whatever the workspace
    bad = list(args); bad[2] = 5
    assert lib.wq_gemm_w4ax_ws(*bad, FAKE, ws(n), None) == 4


@pytest.mark.parametrize("M,K,N,splits", [
    (16, 2048, 512, False),    # short K loop: unsplit
    (16, 4096, 512, True),     # narrow tiles from K = 4096 on
    (128, 4096, 512, False),   # wider tiles split only from K = 8192 on
    (256, 8192, 2048, True),
    (4288, 8192, 2048, False),  # enough output tiles to fill the GPU
    (16, 16384, 4096, True)])
def test_split_rule_on_host(lib, M, K, N, splits):
    """K is split (scratch needed) only for few output tiles with a long K loop."""
    lib.wq_gemm_scratch_bytes.restype = ctypes.c_size_t
    assert (lib.wq_gemm_scratch_bytes(M, K, N) > 0) == splits


def test_static_clipping_entry_points_reject_on_host(lib):
    # wq_act_quant_static(x, M, K, cinv, sid, thr, gain, S, T, step, bits, qx, s_tok, st)
    assert lib.wq_act_quant_static(FAKE, 8, 256, None, FAKE, None, FAKE, 3, 1, 0, 8, FAKE, FAKE,
                                   None) == 1        # no thresholds
    assert lib.wq_act_quant_static(FAKE, 8, 256, None, FAKE, FAKE, None, 3, 1, 0, 8, FAKE, FAKE,
                                   None) == 1        # no gains
    assert lib.wq_act_quant_static(FAKE, 8, 256, None, FAKE, FAKE, FAKE, 3, 1, 0, 6, FAKE, FAKE,
                                   None) == 4        # bits
    assert lib.wq_act_quant_static(FAKE, 8, 200, None, FAKE, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE,
                                   None) == 2        # K
    assert lib.wq_act_quant_static(FAKE, 8, 256, None, FAKE, FAKE, FAKE, 3, 2, 2, 8, FAKE, FAKE,
                                   None) == 4        # step outside the table
    # wq_linear_w4ax_static(x, M, K, N, cinv, sid, thr, gain, beta, S, T, step, bits, qw, s_w,
    #                       bias, y, ws, ws_bytes, st)
    args = [FAKE, 64, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, FAKE, FAKE,
            FAKE, 1 << 30, None]
    bad = list(args); bad[6] = None
    assert lib.wq_linear_w4ax_static(*bad) == 1      # no thresholds
    bad = list(args); bad[7] = None
    assert lib.wq_linear_w4ax_static(*bad) == 1      # no gains
    bad = list(args); bad[12] = 5
    assert lib.wq_linear_w4ax_static(*bad) == 4      # bits
    bad = list(args); bad[18] = 100
    assert lib.wq_linear_w4ax_static(*bad) == 4      # workspace too small


def test_single_kernel_linear_rejects_on_host(lib):
    # (x, M, K, N, cinv, sid, table, thr, beta, S, T, step, bits, qw, s_w, bias, y, st)
    args = [FAKE, 64, 256, 256, FAKE, FAKE, FAKE, None, FAKE, 3, 1, 0, 8, FAKE, FAKE, FAKE, FAKE,
            None]
    bad = list(args); bad[1] = 65
    assert lib.wq_linear_w4ax_single(*bad) == 2      # more tokens than one tile
    bad = list(args); bad[6] = None
    assert lib.wq_linear_w4ax_single(*bad) == 1      # no clip table
    bad = list(args); bad[12] = 6
    assert lib.wq_linear_w4ax_single(*bad) == 4      # bits
    bad = list(args); bad[0] = MIS
    assert lib.wq_linear_w4ax_single(*bad) == 3      # misaligned x
    bad = list(args); bad[1] = 0
    assert lib.wq_linear_w4ax_single(*bad) == 0      # empty batch: nothing to do


def test_every_pointer_is_checked_for_alignment(lib):
    """A table, stream-id or scale pointer off a 16-byte boundary is rejected like the others."""
    # wq_act_quant(x, M, K, cinv, sid, alpha, S, T, step, bits, qx, s_tok, st)
    aq = [FAKE, 8, 256, None, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, None]
    for i in (4, 5, 11):                   # stream_id, alpha, s_tok
        bad = list(aq); bad[i] = MIS
        assert lib.wq_act_quant(*bad) == 3, i
    # wq_act_quant_static(x, M, K, cinv, sid, thr, gain, S, T, step, bits, qx, s_tok, st)
    st = [FAKE, 8, 256, None, FAKE, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, None]
    for i in (4, 5, 6, 12):                # stream_id, thr, gain, s_tok
        bad = list(st); bad[i] = MIS
        assert lib.wq_act_quant_static(*bad) == 3, i
    for kw in (dict(sid=MIS), dict(alpha=MIS)):
        assert _linear(lib, **kw) == 3, kw
    # wq_linear_w4ax_static: thr (index 6) and gain (index 7)
    ls = [FAKE, 64, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, FAKE, FAKE,
          FAKE, 1 << 30, None]
    for i in (5, 6, 7):
        bad = list(ls); bad[i] = MIS
        assert lib.wq_linear_w4ax_static(*bad) == 3, i
    # wq_linear_w4ax_single: stream_id, table, thr
    one = [FAKE, 64, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, FAKE, FAKE,
           None]
    for i in (5, 6, 7):
        bad = list(one); bad[i] = MIS
        assert lib.wq_linear_w4ax_single(*bad) == 3, i
    # wq_gemm_w4ax(qx, s_tok, bits, M, K, N, sid, beta, S, T, step, qw, s_w, bias, y, st)
    gm = [FAKE, FAKE, 8, 16, 128, 32, FAKE, None, 3, 1, 0, FAKE, FAKE, None, FAKE, None]
    for i in (0, 1, 6, 11, 12, 14):
        bad = list(gm); bad[i] = MIS
        assert lib.wq_gemm_w4ax(*bad) == 3, i
    # wq_channel_scale(x_cal, Mcal, W, N, K, c, cinv, st)
    cs = [FAKE, 4, FAKE, 4, 128, FAKE, FAKE, None]
    for i in (0, 2, 5, 6):
        bad = list(cs); bad[i] = MIS
        assert lib.wq_channel_scale(*bad) == 3, i


def _gelu(lib, **kw):
    # (x, M, K, N, cinv, sid, alpha, beta, S, T, step, bits, qw, s_w, bias, cinv_next,
    #  thr_next, gain_next, bits_next, codes, s_next, h, ws, ws_bytes, st)
    a = dict(x=FAKE, M=64, K=256, N=256, cinv=FAKE, sid=FAKE, alpha=FAKE, beta=FAKE, S=3, T=1,
             step=0, bits=8, qw=FAKE, s_w=FAKE, bias=FAKE, cinv_next=FAKE, thr=FAKE, gain=FAKE,
             bits_next=8, codes=FAKE, s_next=FAKE, h=None, ws=FAKE, ws_bytes=1 << 30, st=None)
    a.update(kw)
    return lib.wq_linear_gelu_quant(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(bits_next=6), 4), (dict(bits=5), 4), (dict(thr=None), 1), (dict(gain=None), 1),
    (dict(s_next=None), 1), (dict(codes=None), 1), (dict(codes=MIS), 3), (dict(h=MIS), 3),
    (dict(cinv_next=MIS), 3), (dict(s_next=MIS), 3), (dict(N=250), 2), (dict(ws_bytes=10), 4),
    (dict(step=1), 4), (dict(M=0, x=None, sid=None, codes=None, s_next=None), 0),
])
def test_gelu_quant_rejects_bad_arguments_on_host(lib, kw, code):
    assert _gelu(lib, **kw) == code


def test_debug_linear_rejects_on_host(lib):
    # (x, M, K, N, cinv, sid, alpha, beta, S, T, step, bits, qw, s_w, bias, y, acc, ws, ws_bytes, st)
    args = [FAKE, 64, 256, 256, FAKE, FAKE, FAKE, FAKE, 3, 1, 0, 8, FAKE, FAKE, FAKE, FAKE, FAKE,
            FAKE, 1 << 30, None]
    bad = list(args); bad[16] = None
    assert lib.wq_debug_linear_s32(*bad) == 1        # no accumulator buffer
    bad = list(args); bad[16] = MIS
    assert lib.wq_debug_linear_s32(*bad) == 3
    bad = list(args); bad[11] = 2
    assert lib.wq_debug_linear_s32(*bad) == 4


def test_stall_hook_needs_a_limit(lib):
    assert lib.wq_debug_inject_stall(1, 0) == 4


def test_noalloc_scratch_limit_is_exact(lib):
    """wq_workspace_bytes(M, K, N, 8) <= 16 MiB is the rule: at K = N = 4096 the
    largest M is 4092 (16 MiB exactly); M = 4093 is rejected before any launch."""
    limit = 16 << 20
    assert wq.wq_workspace_bytes(4092, 4096, 4096, 8) == limit
    assert wq.wq_workspace_bytes(4093, 4096, 4096, 8) > limit
    args = lambda m: (FAKE, m, 4096, 4096, None, FAKE, FAKE, None, 3, 1, 0, FAKE, FAKE, None,
                      FAKE, None)
    assert wq.STATUS[lib.wq_linear_w4a8_noalloc(*args(4093))] == "WQ_ERR_SCRATCH"
    # 4092 passes the size check; without a GPU the next step (finding the device) fails
    assert wq.STATUS[lib.wq_linear_w4a8_noalloc(*args(4092))] != "WQ_ERR_SCRATCH"


# ------------------------------------------------------------------ the GEMM's launch plan
# wq_gemm_plan_query reports which GEMM instance a call runs for a shape (host
# arithmetic only).  The hidden-4096 block takes 224-token CTA pairs for all four
# linears; at 4288 tokens, 224-token tiles would give the busiest of the 74 pairs
# more token columns on qkv, attn_out and mlp_down than 256-token tiles do.
BLOCK4096 = [(8512, 4096, 12288), (8512, 4096, 4096), (8512, 4096, 16384), (8512, 16384, 4096)]
BLOCK2048 = [(4288, 2048, 6144), (4288, 2048, 2048), (4288, 2048, 8192), (4288, 8192, 2048)]


@pytest.mark.parametrize("M,K,N,tile", [(*s, 224) for s in BLOCK4096] +
                         list(zip(*zip(*BLOCK2048), (256, 256, 224, 256))))
def test_plan_of_the_configured_blocks(lib, M, K, N, tile):
    p = wq.wq_gemm_plan_query(M, K, N)
    assert (p["tile_tokens"], p["tile_channels"], p["ctas_per_tile"]) == (tile, 256, 2)
    assert p["k_splits"] == 1 and p["k_stage"] == 128
    assert p["weights_in_tmem"] == (tile == 224)
    assert p["tiles"] == -(-M // tile) * (N // 256)
    # the GELU-and-quantize epilogue keeps 256-token pairs with the weights in shared memory
    g = wq.wq_gemm_plan_query(M, K, N, call="gelu_quant")
    assert (g["tile_tokens"], g["ctas_per_tile"], g["weights_in_tmem"]) == (256, 2, 0)


def _busiest(M, N, bn, pairs=74):
    tiles = -(-N // 256) * -(-M // bn)
    return -(-tiles // pairs) * bn


@pytest.mark.parametrize("M", [129, 200, 256, 300, 513, 1000, 2048, 4288, 6000, 8512])
@pytest.mark.parametrize("N", [256, 2048, 4096, 6144, 12288])
def test_pair_width_balances_the_pairs(lib, M, N):
    """Pair tiles take 224 tokens unless that leaves the busiest pair more token
    columns than 256 does (whole tiles per pair; 148 SMs without a device)."""
    p = wq.wq_gemm_plan_query(M, 4096, N, call="gemm")
    assert p["ctas_per_tile"] == 2
    want = 224 if _busiest(M, N, 224) <= _busiest(M, N, 256) else 256
    assert p["tile_tokens"] == want


@pytest.mark.parametrize("M", [1, 16, 33, 64, 100, 128, 256, 300])
@pytest.mark.parametrize("K,N", [(2048, 512), (4096, 384), (8192, 2048), (16384, 4096),
                                 (384, 256)])
@pytest.mark.parametrize("act_bits", [8, 4])
def test_plan_agrees_with_the_scratch_rule(lib, M, K, N, act_bits):
    """K is split exactly when the call takes a scratch and wq_gemm_scratch_bytes is
    not 0; split shapes and packed int4 codes run single CTAs; 256-deep stages only
    for tiles of at most 64 tokens with K a multiple of 256."""
    lib.wq_gemm_scratch_bytes.restype = ctypes.c_size_t
    split = lib.wq_gemm_scratch_bytes(M, K, N) > 0
    for call in ("gemm", "gemm_ws", "linear"):
        bits = 8 if call == "linear" else act_bits
        p = wq.wq_gemm_plan_query(M, K, N, act_bits, call)
        assert (p["k_splits"] > 1) == (split and call != "gemm")
        pair = p["ctas_per_tile"] == 2
        assert pair == (bits == 8 and M > 128 and p["k_splits"] == 1)
        assert p["tile_channels"] == (256 if pair else 128)
        if not pair:
            assert p["tile_tokens"] == next((b for b in (16, 32, 64, 128) if M <= b), 256)
        assert p["k_stage"] == (256 if p["tile_tokens"] <= 64 and K % 256 == 0 else 128)
        assert p["weights_in_tmem"] == (p["k_stage"] == 256 or p["tile_tokens"] == 224)
        assert p["tiles"] == -(-M // p["tile_tokens"]) * -(-N // p["tile_channels"])


def test_plan_rejects_on_host(lib):
    plan = wq.GemmPlan()
    q = lib.wq_gemm_plan_query
    assert q(16, 4096, 512, 8, 0, None) == 1                      # no plan
    assert q(16, 4096, 512, 8, 4, ctypes.byref(plan)) == 4        # unknown call
    assert q(16, 4096, 512, 5, 0, ctypes.byref(plan)) == 4        # bad act_bits
    assert q(16, 4096, 512, 5, 2, ctypes.byref(plan)) == 0        # ignored for the linears
    assert q(16, 100, 512, 8, 2, ctypes.byref(plan)) == 2         # K not a multiple of 128
    assert q(16, 4096, 8, 8, 2, ctypes.byref(plan)) == 2          # N below 16
    plan.tiles = 7
    assert q(0, 4096, 512, 8, 2, ctypes.byref(plan)) == 0 and plan.tiles == 0  # empty batch


def test_plan_call_names_match_the_header():
    src = open(os.path.join(ROOT, "include", "wq.h")).read()
    enum = {m.group(1).lower(): int(m.group(2))
            for m in re.finditer(r"\bWQ_PLAN_([A-Z_]+)\s*=\s*(\d+)", src)}
    assert enum == wq.PLAN_CALLS


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++17")])
def test_header_is_plain_c(lang, std):
    """include/wq.h is a C header (plain pointers, sizes and enums; no CUDA or torch
    types): it compiles as strict C99 and as C++, with every warning an error."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = ('#include "wq.h"\n'
           "int main(void) { wq_gemm_plan p; wq_stream_t s = 0; (void)s; p.tiles = 0;\n"
           "  return p.tiles + (int)WQ_PLAN_LINEAR + (int)WQ_ERR_SCRATCH; }\n")
    r = subprocess.run([cc, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), "-x", lang, "-"],
                       input=src, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
