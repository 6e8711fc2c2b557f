"""The C-ABI library on the CPU: it loads, exports every symbol include/zmoe.h declares, and rejects
bad arguments on the host (no compute call is made: nothing here needs a GPU)."""
import ctypes
import os
import re

import pytest

from sparse_moe_decoder_b200 import build as B
from sparse_moe_decoder_b200 import zmoe as Z

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "zmoe.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return Z.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ZMOE_API\s+[\w\s\*]+?\b(zmoe_\w+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("zmoe_delay_shear", "zmoe_delay_unshear", "zmoe_embed_sum_rmsnorm", "zmoe_route", "zmoe_permute",
              "zmoe_grouped_swiglu", "zmoe_combine"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), f"libzmoe.so does not export {n}"
        assert n in Z.SIGNATURES, f"the binding has no signature for {n}"


def test_status_strings_and_version(L):
    assert L.zmoe_version() >= 100
    assert L.zmoe_status_string(0) == b"ok"
    assert L.zmoe_status_string(1) == b"invalid argument"
    assert L.zmoe_status_string(99) == b"unknown status"


NULL = None


@pytest.mark.parametrize("call", [
    lambda L: L.zmoe_delay_shear(NULL, NULL, 1, 4, 0, 1024, NULL),              # N = 0
    lambda L: L.zmoe_delay_shear(NULL, NULL, 1, 4, 9, 1024, NULL),              # NULL pointers
    lambda L: L.zmoe_delay_unshear(NULL, NULL, 1, 3, 9, NULL),                  # Ty < N - 1
    lambda L: L.zmoe_embed_sum_rmsnorm(NULL, NULL, 1, NULL, 1e-6, 2, 9, 1025, 12, NULL, 1, NULL),  # d % 8
    lambda L: L.zmoe_embed_sum_rmsnorm(NULL, NULL, 7, NULL, 1e-6, 2, 9, 1025, 16, NULL, 1, NULL),  # dtype
    lambda L: L.zmoe_rmsnorm(NULL, 0, NULL, -1.0, 2, 16, NULL, 0, NULL),       # eps < 0
    lambda L: L.zmoe_route(NULL, NULL, 1, NULL, NULL, 4, 64, 16, 3, NULL, NULL, NULL, NULL),   # k = 3
    lambda L: L.zmoe_route(NULL, NULL, 1, NULL, NULL, 4, 64, 65, 1, NULL, NULL, NULL, NULL),   # E = 65
    lambda L: L.zmoe_route(NULL, NULL, 1, NULL, NULL, 4, 64, 1, 2, NULL, NULL, NULL, NULL),    # k > E
    lambda L: L.zmoe_route(NULL, NULL, 1, NULL, NULL, 4, 64, 16, 1, NULL, NULL, NULL, NULL),   # NULL
    lambda L: L.zmoe_permute(NULL, NULL, 1, 4, 64, 16, 1, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL),
    lambda L: L.zmoe_grouped_swiglu(NULL, NULL, 4, NULL, NULL, NULL, 1, 16, 64, 64, NULL, NULL, NULL, 0, NULL),
    lambda L: L.zmoe_combine(NULL, NULL, NULL, NULL, 4, 64, 3, NULL, NULL),    # k = 3
    lambda L: L.zmoe_combine(NULL, NULL, NULL, NULL, 4, 6, 1, NULL, NULL),     # d % 4
    lambda L: L.zmoe_moe_layer(NULL, NULL, NULL, 1e-6, NULL, NULL, NULL, NULL, NULL, NULL, 1, 4, 256, 256, 16, 3,
                               NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL),     # k = 3
    lambda L: L.zmoe_moe_layer(NULL, NULL, NULL, 1e-6, NULL, NULL, NULL, NULL, NULL, NULL, 1, 4, 256, 256, 16, 1,
                               NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL),     # no router with E = 16
    lambda L: L.zmoe_output_heads(NULL, NULL, 1e-6, NULL, 1, 2, 9, 1025, 12, NULL, NULL, NULL, NULL, 0, NULL),  # d % 8
    lambda L: L.zmoe_output_heads(NULL, NULL, 1e-6, NULL, 1, 2, 9, 1025, 16, NULL, NULL, NULL, NULL, 0, NULL),  # NULL
    lambda L: L.zmoe_speaker_prefix(NULL, NULL, 1, NULL, 2, 2048, 1020, NULL, NULL),   # n_in % 8
    lambda L: L.zmoe_speaker_prefix(NULL, NULL, 1, NULL, 2, 2048, 1024, NULL, NULL),   # NULL
])
def test_bad_arguments_rejected_on_host(L, call):
    assert call(L) == 1   # ZMOE_ERR_INVALID_ARG, nothing launched
    assert len(L.zmoe_last_error()) > 0


def _fp8_layer(L, T=4, d=256, f=256, E=16, k=1, x=0x1000, h=NULL, gamma=NULL, w_router=0x2000, q_gate=0x3000,
               y=0x4000):
    """zmoe_moe_layer_fp8 with placeholder (never dereferenced) 16-byte-aligned pointers by default."""
    s = 0x5000
    return L.zmoe_moe_layer_fp8(x, h, gamma, 1e-6, w_router, NULL, NULL, q_gate, s, 0x6000, s, 0x7000, s, T, d, f, E,
                                k, y, NULL, NULL, NULL, NULL, NULL, 0, NULL)


@pytest.mark.parametrize("kw", [
    dict(T=-1), dict(E=65), dict(E=0), dict(k=3), dict(k=2, E=1), dict(d=384), dict(f=128),
    dict(q_gate=NULL), dict(y=NULL), dict(w_router=NULL),          # no router with E = 16
    dict(x=NULL), dict(gamma=0x8000),                              # neither x nor h with gamma
])
def test_fp8_layer_bad_arguments_rejected_on_host(L, kw):
    assert _fp8_layer(L, **kw) == 1   # ZMOE_ERR_INVALID_ARG, nothing launched
    assert len(L.zmoe_last_error()) > 0


def test_fp8_layer_unaligned_and_empty(L):
    assert _fp8_layer(L, q_gate=0x3000 + 8) == 1
    assert b"aligned" in L.zmoe_last_error()
    assert _fp8_layer(L, T=0) == 0     # nothing to do: OK without touching the device


def test_unaligned_pointers_rejected(L):
    # 16-byte alignment is checked on the host before any launch (pointer values are never dereferenced)
    p = ctypes.c_void_p(0x1000 + 4)
    q = ctypes.c_void_p(0x2000)
    st = L.zmoe_route(p, q, 1, NULL, NULL, 4, 64, 16, 1, q, q, NULL, NULL)
    assert st == 1
    assert b"aligned" in L.zmoe_last_error()


def test_empty_problems_are_no_ops(L):
    # nothing to do -> OK without touching the device
    assert L.zmoe_route(NULL, NULL, 1, NULL, NULL, 0, 64, 16, 1, NULL, NULL, NULL, NULL) == 0
    assert L.zmoe_combine(NULL, NULL, NULL, NULL, 0, 64, 1, NULL, NULL) == 0
    assert L.zmoe_delay_shear(NULL, NULL, 0, 5, 9, 1024, NULL) == 0


def test_empty_new_entry_points_are_no_ops(L):
    assert L.zmoe_moe_layer(NULL, NULL, NULL, 1e-6, NULL, NULL, NULL, NULL, NULL, NULL, 1, 0, 256, 256, 16, 1,
                            NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == 0
    assert L.zmoe_output_heads(NULL, NULL, 1e-6, NULL, 1, 0, 9, 1025, 2048, NULL, NULL, NULL, NULL, 0, NULL) == 0
    assert L.zmoe_speaker_prefix(NULL, NULL, 1, NULL, 0, 2048, 1024, NULL, NULL) == 0
    assert L.zmoe_output_heads_workspace_size(0, 9) >= 0 and L.zmoe_output_heads_workspace_size(4, 9) >= 4 * 9 * 8


def test_workspace_queries(L):
    assert L.zmoe_permute_workspace_size(16384, 16, 2) >= (32768 // 256) * 16 * 4
    assert L.zmoe_permute_workspace_size(-1, 16, 1) == 0
    assert L.zmoe_grouped_swiglu_workspace_size(64, 16, 2048, 3072, 1) >= 0


def test_layer_dispatch_by_batch_size(L):
    """zmoe_moe_layer's launch choice, visible in its workspace query (host logic, no device call made
    beyond the attribute queries): T * k <= 4 takes the tiny-batch launch, whose workspace is one
    256-byte counter block plus h in fp32 for the T k assignments; larger decode batches take the
    stream-K launch, with its per-SM partial slots."""
    BF16 = 1   # ZMOE_BF16
    for T, k in [(1, 1), (1, 2), (2, 2), (4, 1)]:
        assert L.zmoe_moe_layer_workspace_size(T, 2048, 3072, 16, k, BF16) == 256 + T * k * 3072 * 4
    big = L.zmoe_moe_layer_workspace_size(5, 2048, 3072, 16, 1, BF16)
    assert big > 256 + 5 * 3072 * 4 + 148 * 2 * 2 * 16 * 128 * 4



def test_timeout_injection_checks_its_limit(L):
    """The test hook of the timeout path only sets host-side state: no GPU needed."""
    assert L.zmoe_debug_inject_timeout(1, 10) == 1                  # below 1 us: ZMOE_ERR_INVALID_ARG
    assert L.zmoe_debug_inject_timeout(1, 3_000_000_000) == 1       # above 2 s
    assert L.zmoe_debug_inject_timeout(0, 0) == 0


# Placeholder device pointers: 16-byte aligned, never dereferenced (every case fails on the host first).
_A, _B, _C, _D, _S = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000


def _w8a8_layer(L, T=4, d=256, f=256, E=16, k=1, x=_A, h=NULL, gamma=NULL, w_router=_B, q_gate=_C, s_gate=_S,
                y=_D):
    return L.zmoe_moe_layer_w8a8(x, h, gamma, 1e-6, w_router, NULL, NULL, q_gate, s_gate, _C, _S, _C, _S, T, d, f, E,
                                 k, y, NULL, NULL, NULL, NULL, NULL, 0, NULL)


@pytest.mark.parametrize("kw", [
    dict(T=-1), dict(E=65), dict(k=3), dict(k=2, E=1), dict(d=384), dict(f=128), dict(q_gate=NULL), dict(y=NULL),
    dict(w_router=NULL), dict(x=NULL), dict(gamma=_S), dict(s_gate=_S + 4),
])
def test_w8a8_layer_bad_arguments_rejected_on_host(L, kw):
    assert _w8a8_layer(L, **kw) == 1
    assert len(L.zmoe_last_error()) > 0


def _f16h_layer(L, T=4, d=256, f=256, E=16, k=1, x=_A, w_down_f16=_C, down_scale=_S, y=_D):
    return L.zmoe_moe_layer_f16h(x, NULL, NULL, 1e-6, _B, NULL, NULL, _C, _C, w_down_f16, down_scale, T, d, f, E, k, y,
                                 NULL, NULL, NULL, NULL, NULL, 0, NULL)


@pytest.mark.parametrize("kw", [
    dict(T=-1), dict(E=0), dict(k=3), dict(d=2056), dict(f=264), dict(w_down_f16=NULL), dict(down_scale=NULL),
    dict(x=_A + 8),
])
def test_f16h_layer_bad_arguments_rejected_on_host(L, kw):
    assert _f16h_layer(L, **kw) == 1
    assert len(L.zmoe_last_error()) > 0


@pytest.mark.parametrize("args", [
    dict(M=-1), dict(E=65), dict(d=200), dict(offsets=NULL), dict(h=NULL), dict(h=_D + 2),
])
def test_grouped_swiglu_f16h_bad_arguments_rejected_on_host(L, args):
    a = dict(M=64, E=4, d=256, f=256, offsets=_S, h=_D)
    a.update(args)
    assert L.zmoe_grouped_swiglu_f16h(_A, a["offsets"], a["M"], _B, _B, _C, _S, a["E"], a["d"], a["f"], a["h"], _D,
                                      NULL) == 1
    assert len(L.zmoe_last_error()) > 0


def test_prepare_w_down_f16_checks_its_arguments_and_workspace(L):
    assert L.zmoe_prepare_w_down_f16(_A, 0, 256, 256, _B, _S, _C, 64, NULL) == 1        # E = 0
    assert L.zmoe_prepare_w_down_f16(_A, 4, 252, 256, _B, _S, _C, 64, NULL) == 1        # d % 8
    assert L.zmoe_prepare_w_down_f16(_A, 4, 256, 256, NULL, _S, _C, 64, NULL) == 1      # NULL output
    assert L.zmoe_prepare_w_down_f16(_A + 8, 4, 256, 256, _B, _S, _C, 64, NULL) == 1    # unaligned
    assert L.zmoe_prepare_w_down_f16(_A, 16, 256, 256, _B, _S, _C, 63, NULL) == 4       # 4 E bytes needed
    assert b"workspace" in L.zmoe_last_error()


def _stack_layers(n, **over):
    arr = (Z.StackLayer * n)()
    for i in range(n):
        f = dict(w_router=_A, logit_bias=NULL, sel_bias=NULL, gamma=_S, w_gate=_B, w_up=_C, w_down=_D, E=16, k=1)
        f.update(over)
        arr[i] = Z.StackLayer(f["w_router"], f["logit_bias"], f["sel_bias"], f["gamma"], f["w_gate"], f["w_up"],
                              f["w_down"], f["E"], f["k"])
    return arr


@pytest.mark.parametrize("case", [
    dict(n=0), dict(n=33), dict(d=2044), dict(d=4104), dict(f=3070), dict(eps=-1.0), dict(h=NULL), dict(h=_D + 4),
    dict(ids=_S, N=0), dict(ids=_S, N=33), dict(layer=dict(E=65)), dict(layer=dict(k=3)), dict(layer=dict(E=1, k=2)),
    dict(layer=dict(w_router=NULL)), dict(layer=dict(w_down=NULL)), dict(layer=dict(w_gate=_B + 8)),
])
def test_decode_stack_bad_arguments_rejected_on_host(L, case):
    n = case.get("n", 2)
    arr = _stack_layers(max(n, 1), **case.get("layer", {}))
    st = L.zmoe_decode_stack(ctypes.cast(arr, ctypes.c_void_p), n, case.get("d", 2048), case.get("f", 3072),
                             case.get("eps", 1e-6), case.get("ids", NULL), _A, _S, case.get("N", 9), 1025,
                             case.get("h", _D), NULL, NULL, NULL, NULL, _C, 1 << 20, NULL)
    assert st == 1
    assert len(L.zmoe_last_error()) > 0
