"""The Python binding's marshalling, on a machine without a GPU: a fake library
records what each wrapper would pass to its C entry point, and fake device tensors
stand in for CUDA tensors.  Checks that every wrapper passes sizes and addresses
in the order include/wq.h declares, and that a tensor the C call would read or
write past its end, of the wrong element type, on the host or on another device
is rejected before any call."""
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq


class DevT:
    """Shape, type and a made-up address of a device tensor; never dereferenced."""
    _next = 1 << 24

    def __init__(self, shape, dtype, device=0, contiguous=True, cuda=True):
        self._t = torch.empty(shape, dtype=dtype)
        self.addr = DevT._next
        DevT._next += 1 << 16
        self.device, self.contiguous, self.is_cuda = device, contiguous, cuda

    shape = property(lambda self: self._t.shape)
    dtype = property(lambda self: self._t.dtype)

    def numel(self):
        return self._t.numel()

    def element_size(self):
        return self._t.element_size()

    def is_contiguous(self):
        return self.contiguous

    def get_device(self):
        return self.device

    def data_ptr(self):
        return self.addr


class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append((name, args))
            return 0
        return f


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(wq, "_lib", lib)
    monkeypatch.setattr(wq, "_current_device", lambda: 0)
    return lib


M, K, N, S, T, STEP = 40, 256, 48, 3, 2, 1
F32, BF16 = torch.float32, torch.bfloat16


def tensors(bits=8, x_dtype=BF16):
    return dict(
        x=DevT((M, K), x_dtype), cinv=DevT((K,), F32), sid=DevT((M,), torch.uint8),
        alpha=DevT((T, S), F32), beta=DevT((T, S, N), F32), thr=DevT((T,), F32),
        qw=DevT((N, K // 2), torch.uint8), s_w=DevT((N,), F32), bias=DevT((N,), F32),
        y=DevT((M, N), BF16), s_tok=DevT((M,), F32),
        qx=DevT((M, K) if bits == 8 else (M, K // 2), torch.int8 if bits == 8 else torch.uint8),
        ws=DevT((wq_ws_bytes(bits),), torch.uint8), acc=DevT((M, N), torch.int32))


def wq_ws_bytes(bits):
    return M * K + 4096   # any size: the library checks it against wq_workspace_bytes()


def p(t):
    return t.addr


@pytest.mark.parametrize("x_dtype", [BF16, torch.int16, torch.uint16])
def test_linear_marshals_in_header_order(fake, x_dtype):
    a = tensors(x_dtype=x_dtype)
    wq.wq_linear_w4a8(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, a["qw"],
                      a["s_w"], a["bias"], a["y"], a["ws"], stream=0)
    (name, args), = fake.calls
    assert name == "wq_linear_w4a8"
    assert args == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["alpha"]), p(a["beta"]),
                    S, T, STEP, p(a["qw"]), p(a["s_w"]), p(a["bias"]), p(a["y"]), p(a["ws"]),
                    wq_ws_bytes(8), 0)


def test_every_other_wrapper_marshals_in_header_order(fake):
    a = tensors()
    a4 = tensors(bits=4)
    W, xc = DevT((N, K), torch.int16), DevT((7, K), torch.int16)
    c = DevT((K,), F32)
    wq.wq_channel_scale(xc, W, c, a["cinv"], stream=0)
    wq.wq_pack_int4(W, c, a["qw"], a["s_w"], stream=0)
    wq.wq_act_quant(a["x"], a["cinv"], a["sid"], a["alpha"], STEP, 8, a["qx"], a["s_tok"], 0)
    wq.wq_act_quant(a4["x"], None, a4["sid"], a4["alpha"], STEP, 4, a4["qx"], a4["s_tok"], 0)
    wq.wq_act_quant_static(a["x"], a["cinv"], a["sid"], a["thr"], a["alpha"], STEP, 8, a["qx"],
                           a["s_tok"], 0)
    wq.wq_gemm_w4ax(a4["qx"], a["s_tok"], 4, K, a["sid"], None, S, T, STEP, a["qw"], a["s_w"],
                    None, a["y"], 0)
    wq.wq_linear_w4a4(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, a["qw"],
                      a["s_w"], a["bias"], a["y"], a["ws"], stream=0)
    wq.wq_linear_w4ax_static(a["x"], a["cinv"], a["sid"], a["thr"], a["alpha"], a["beta"], STEP,
                             4, a["qw"], a["s_w"], a["bias"], a["y"], a["ws"], stream=0)
    wq.wq_linear_w4ax_single(a["x"], a["cinv"], a["sid"], a["alpha"], None, a["beta"], STEP, 8,
                             a["qw"], a["s_w"], a["bias"], a["y"], stream=0)
    wq.wq_linear_w4a8_noalloc(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, a["qw"],
                              a["s_w"], a["bias"], a["y"], stream=0)
    wq.wq_debug_gemm_s32(a["qx"], 8, a["qw"], K, a["acc"], a["ws"], stream=0)
    wq.wq_debug_linear_s32(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, 4, a["qw"],
                           a["s_w"], a["bias"], a["y"], a["acc"], a["ws"], stream=0)
    codes, s_next, h = DevT((M, N), torch.int8), DevT((M,), F32), DevT((M, N), BF16)
    cinv_n, gain_n = DevT((N,), F32), DevT((T, S), F32)
    wq.wq_linear_gelu_quant(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, 8, a["qw"],
                            a["s_w"], a["bias"], cinv_n, a["thr"], gain_n, 4, codes, s_next, h,
                            a["ws"], stream=0)
    wq.wq_debug_inject_stall(True, 50000)
    got = dict((n, args) for n, args in fake.calls[:2])
    assert got["wq_channel_scale"] == (p(xc), 7, p(W), N, K, p(c), p(a["cinv"]), 0)
    assert got["wq_pack_int4"] == (p(W), p(c), N, K, p(a["qw"]), p(a["s_w"]), 0)
    rest = [args for _, args in fake.calls[2:]]
    assert [n for n, _ in fake.calls[2:]] == [
        "wq_act_quant", "wq_act_quant", "wq_act_quant_static", "wq_gemm_w4ax", "wq_linear_w4a4",
        "wq_linear_w4ax_static", "wq_linear_w4ax_single", "wq_linear_w4a8_noalloc",
        "wq_debug_gemm_s32", "wq_debug_linear_s32", "wq_linear_gelu_quant",
        "wq_debug_inject_stall"]
    assert rest[0] == (p(a["x"]), M, K, p(a["cinv"]), p(a["sid"]), p(a["alpha"]), S, T, STEP, 8,
                       p(a["qx"]), p(a["s_tok"]), 0)
    assert rest[1] == (p(a4["x"]), M, K, None, p(a4["sid"]), p(a4["alpha"]), S, T, STEP, 4,
                       p(a4["qx"]), p(a4["s_tok"]), 0)
    assert rest[2] == (p(a["x"]), M, K, p(a["cinv"]), p(a["sid"]), p(a["thr"]), p(a["alpha"]),
                       S, T, STEP, 8, p(a["qx"]), p(a["s_tok"]), 0)
    assert rest[3] == (p(a4["qx"]), p(a["s_tok"]), 4, M, K, N, p(a["sid"]), None, S, T, STEP,
                       p(a["qw"]), p(a["s_w"]), None, p(a["y"]), 0)
    assert rest[4] == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["alpha"]),
                       p(a["beta"]), S, T, STEP, p(a["qw"]), p(a["s_w"]), p(a["bias"]),
                       p(a["y"]), p(a["ws"]), wq_ws_bytes(8), 0)
    assert rest[5] == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["thr"]),
                       p(a["alpha"]), p(a["beta"]), S, T, STEP, 4, p(a["qw"]), p(a["s_w"]),
                       p(a["bias"]), p(a["y"]), p(a["ws"]), wq_ws_bytes(8), 0)
    assert rest[6] == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["alpha"]), None,
                       p(a["beta"]), S, T, STEP, 8, p(a["qw"]), p(a["s_w"]), p(a["bias"]),
                       p(a["y"]), 0)
    assert rest[7] == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["alpha"]),
                       p(a["beta"]), S, T, STEP, p(a["qw"]), p(a["s_w"]), p(a["bias"]),
                       p(a["y"]), 0)
    assert rest[8] == (p(a["qx"]), 8, p(a["qw"]), M, N, K, p(a["acc"]), p(a["ws"]),
                       wq_ws_bytes(8), 0)
    assert rest[9] == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["alpha"]),
                       p(a["beta"]), S, T, STEP, 4, p(a["qw"]), p(a["s_w"]), p(a["bias"]),
                       p(a["y"]), p(a["acc"]), p(a["ws"]), wq_ws_bytes(8), 0)
    assert rest[10] == (p(a["x"]), M, K, N, p(a["cinv"]), p(a["sid"]), p(a["alpha"]),
                        p(a["beta"]), S, T, STEP, 8, p(a["qw"]), p(a["s_w"]), p(a["bias"]),
                        p(cinv_n), p(a["thr"]), p(gain_n), 4, p(codes), p(s_next), p(h),
                        p(a["ws"]), wq_ws_bytes(8), 0)
    assert rest[11] == (1, 50000)


@pytest.mark.parametrize("which,bad", [
    ("codes", DevT((M, N - 16), torch.int8)),     # codes smaller than M x N
    ("codes", DevT((M, N), torch.int32)),         # one int8 byte per code
    ("s_next", DevT((M - 1,), F32)),
    ("h", DevT((M, N), F32)),                     # h is bf16
    ("cinv_n", DevT((N - 16,), F32)),             # the next linear's channel scale covers N
    ("gain_n", DevT((T, S - 1), F32)),
])
def test_gelu_quant_rejects_a_bad_tensor_before_the_call(fake, which, bad):
    a = tensors()
    t = dict(codes=DevT((M, N), torch.int8), s_next=DevT((M,), F32), h=DevT((M, N), BF16),
             cinv_n=DevT((N,), F32), gain_n=DevT((T, S), F32))
    t[which] = bad
    with pytest.raises((ValueError, TypeError)):
        wq.wq_linear_gelu_quant(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, 8,
                                a["qw"], a["s_w"], a["bias"], t["cinv_n"], a["thr"], t["gain_n"],
                                8, t["codes"], t["s_next"], t["h"], a["ws"], stream=0)
    assert fake.calls == []


def test_debug_linear_checks_the_accumulator_buffer(fake):
    a = tensors()
    for bad in (DevT((M, N - 16), torch.int32), DevT((M, N), F32)):
        with pytest.raises((ValueError, TypeError)):
            wq.wq_debug_linear_s32(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, 8,
                                   a["qw"], a["s_w"], a["bias"], a["y"], bad, a["ws"], stream=0)
    assert fake.calls == []


def _linear(a):
    wq.wq_linear_w4a8(a["x"], a["cinv"], a["sid"], a["alpha"], a["beta"], STEP, a["qw"],
                      a["s_w"], a["bias"], a["y"], a["ws"], stream=0)


@pytest.mark.parametrize("key,bad,err", [
    ("y", DevT((M, N - 16), BF16), ValueError),            # output smaller than M x N
    ("y", DevT((M, N), torch.float32), TypeError),         # fp32 output: the kernel writes bf16
    ("qw", DevT((N, K // 2 - 64), torch.uint8), ValueError),   # rows shorter than K/2 bytes
    ("s_w", DevT((N,), torch.float16), TypeError),
    ("s_w", DevT((N - 1,), F32), ValueError),
    ("bias", DevT((N // 2,), F32), ValueError),
    ("beta", DevT((T, S, N - 16), F32), ValueError),        # table narrower than N
    ("beta", DevT((T, S, N), BF16), TypeError),
    ("cinv", DevT((K - 128,), F32), ValueError),
    ("sid", DevT((M,), torch.int32), TypeError),
    ("sid", DevT((M - 1,), torch.uint8), ValueError),
    ("x", DevT((M, K), torch.float32), TypeError),
    ("x", DevT((M, K), BF16, cuda=False), ValueError),     # host tensor
    ("x", DevT((M, K), BF16, device=1), ValueError),       # another GPU
    ("y", DevT((M, N), BF16, contiguous=False), ValueError),
    ("ws", DevT((64,), torch.uint8, device=1), ValueError),
])
def test_linear_rejects_a_bad_tensor_before_the_call(fake, key, bad, err):
    a = tensors()
    a[key] = bad
    with pytest.raises(err):
        _linear(a)
    assert fake.calls == []


def test_codes_buffer_is_sized_by_the_code_width(fake):
    a = tensors(bits=4)                       # qx packed: K/2 bytes per row
    wq.wq_act_quant(a["x"], a["cinv"], a["sid"], a["alpha"], STEP, 4, a["qx"], a["s_tok"], 0)
    with pytest.raises(ValueError):           # the same buffer cannot hold int8 codes
        wq.wq_act_quant(a["x"], a["cinv"], a["sid"], a["alpha"], STEP, 8, a["qx"], a["s_tok"], 0)
    with pytest.raises(ValueError):
        wq.wq_gemm_w4ax(a["qx"], a["s_tok"], 8, K, a["sid"], None, S, T, STEP, a["qw"],
                        a["s_w"], None, a["y"], 0)
    with pytest.raises(ValueError):           # acc [M][N+16] needs N+16 weight rows
        wq.wq_debug_gemm_s32(a["qx"], 4, a["qw"], K, DevT((M, N + 16), torch.int32), stream=0)
    assert len(fake.calls) == 1


def test_empty_batch_may_pass_no_token_tensors(fake):
    a = tensors()
    a["x"] = DevT((0, K), BF16)
    a["y"] = DevT((0, N), BF16)
    a["sid"] = None
    _linear(a)
    (name, args), = fake.calls
    assert args[1] == 0 and args[5] is None


def test_library_status_is_raised(monkeypatch):
    class Failing(FakeLib):
        def __getattr__(self, name):
            return lambda *args: 2
    monkeypatch.setattr(wq, "_lib", Failing())
    monkeypatch.setattr(wq, "_current_device", lambda: 0)
    with pytest.raises(wq.WQError, match="WQ_ERR_SHAPE"):
        _linear(tensors())


def test_plan_query_marshals_in_header_order(fake):
    """wq_gemm_plan_query(M, K, N, act_bits, call, plan*): the call's name maps to
    the header's enum, and an unknown name is refused before the library."""
    plan = wq.wq_gemm_plan_query(300, 4096, 512, 4, "gemm_ws")
    name, args = fake.calls[-1]
    assert name == "wq_gemm_plan_query" and args[:5] == (300, 4096, 512, 4, 1)
    assert set(plan) == {"tile_tokens", "tile_channels", "ctas_per_tile", "k_splits",
                         "k_stage", "tiles", "weights_in_tmem"}
    assert [wq.PLAN_CALLS[c] for c in ("gemm", "gemm_ws", "linear", "gelu_quant")] == [0, 1, 2, 3]
    with pytest.raises(KeyError):
        wq.wq_gemm_plan_query(300, 4096, 512, 8, "single")
    assert len(fake.calls) == 1
