"""CPU checks of the C ABI: the library builds for sm_100a, loads, exports
every entry point include/moeq.h declares, sizes records like the oracle, and
rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moeq():
    from quantized_expert_ffn_topk_b200 import build
    build.build()
    import quantized_expert_ffn_topk_b200 as m
    return m


def declared_functions():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            src = open(os.path.join(ROOT, "include", hdr)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^[A-Za-z_][\w \*]*?\b(moe_\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_every_declared_symbol_is_exported(moeq):
    names = declared_functions()
    assert "moe_pack_q" in names and "moe_router_topk" in names
    assert "moe_expert_ffn_q" in names and "moe_combine_residual" in names
    lib = ctypes.CDLL(moeq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    # the binding wraps exactly the declared calls
    assert set(moeq.exported_symbols()) >= set(names)


def test_abi_version_and_status_strings(moeq):
    assert moeq.lib().moe_abi_version() == 1
    for s in range(9):
        assert moeq.status_str(s)


def test_record_sizes_agree_with_oracle(moeq, ref):
    for (H, I, bits, group) in ((4096, 1024, 4, 64), (4096, 1024, 2, 64), (256, 128, 4, 32), (512, 128, 2, 128)):
        assert moeq.moe_expert_bytes(H, I, bits, group) == ref.expert_bytes(H, I, bits, group)
    assert moeq.moe_expert_bytes(4096, 1024, 4, 64) == 7077888
    lay = moeq.moe_expert_layout(4096, 1024, 4, 64)
    # 16-row tiles; one block per group: 32 lanes x 2 k-steps x 8 bytes + 8 x 8 bytes of tables
    assert lay == [64 * 576, 128 * 64 * 576, 16 * 576, 16, 576, 128]
    assert lay[1] + (4096 // 16) * lay[2] == 7077888
    assert moeq.moe_expert_bytes(4096, 1024, 3, 64) == ref.expert_bytes(4096, 1024, 3, 64) == 5505024
    assert moeq.moe_expert_bytes(4096, 1024, 3, 32) == 0  # a 3-bit block pairs k-steps: group >= 64
    assert moeq.moe_expert_layout(4096, 1024, 3, 64)[4] == 32 * 12 + 64
    assert moeq.moe_expert_bytes(4096, 1024, 5, 64) == 0
    assert moeq.moe_expert_bytes(4096, 1000, 4, 64) == 0
    assert moeq.moe_expert_bytes(384, 128, 2, 128) == ref.expert_bytes(384, 128, 2, 128)  # odd H/group is fine


def test_workspace_size(moeq):
    n1 = moeq.moe_workspace_bytes(1, 4, 4096, 1024, 512)
    n32 = moeq.moe_workspace_bytes(32, 4, 4096, 1024, 512)
    assert n1 >= 256 + 512 * 4 + 5 * 1024 * 4 and n32 > n1
    assert moeq.moe_workspace_bytes(0, 4, 4096, 1024, 512) == 0


A = 0x10000  # aligned fake device address: never dereferenced, every call below fails validation first
M = 0x10008  # misaligned


def test_pack_expert_rejects_bad_arguments(moeq):
    L = moeq.lib()
    good = [A] * 9
    assert L.moe_pack_expert(*([None] + good[1:]), 4096, 1024, 4, 64, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_pack_expert(*good, 4096, 1024, 4, 64, None, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_pack_expert(*good, 4096, 1024, 5, 64, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_pack_expert(*good, 4096, 1024, 3, 32, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_pack_expert(*(good[:4] + [M] + good[5:]), 4096, 1024, 4, 64, A, None, None) == moeq.MOE_ERR_ALIGN


def test_pack_rejects_bad_arguments(moeq):
    L = moeq.lib()
    assert L.moe_pack_q(None, A, A, 4, 64, 4, 32, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_pack_q(A, A, A, 4, 64, 5, 32, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_pack_q(A, A, A, 4, 64, 3, 32, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED  # 24-byte rows
    assert L.moe_pack_q(A, A, A, 4, 64, 4, 48, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_pack_q(A, A, A, 4, 48, 4, 16, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_pack_q(A, A, A, 4, 96, 2, 32, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED  # 24-byte rows
    assert L.moe_pack_q(M, A, A, 4, 64, 4, 32, A, A, None, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_pack_q(A, A, A, -1, 64, 4, 32, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_pack_q(A, A, A, 0, 64, 4, 32, A, A, None, None) == moeq.MOE_OK  # nothing to do


def test_router_rejects_bad_arguments(moeq):
    L = moeq.lib()
    ws_n = moeq.moe_workspace_bytes(1, 4, 4096, 1024, 512)
    args = dict(x=A, w=A, B=1, H=4096, E=512, K=4, renorm=0, forced=None, idx=A, wout=A, lg=None, ws=A, n=ws_n)

    def call(**kw):
        a = dict(args, **kw)
        return L.moe_router_topk(a["x"], a["w"], a["B"], a["H"], a["E"], a["K"], a["renorm"], a["forced"], a["idx"],
                                 a["wout"], a["lg"], a["ws"], a["n"], None)
    assert call(x=None) == moeq.MOE_ERR_INVALID_ARG
    assert call(K=9) == moeq.MOE_ERR_INVALID_ARG
    assert call(K=5, E=4) == moeq.MOE_ERR_INVALID_ARG
    assert call(B=0) == moeq.MOE_ERR_INVALID_ARG
    assert call(B=129) == moeq.MOE_ERR_INVALID_ARG
    assert call(ws=None) == moeq.MOE_ERR_WORKSPACE
    assert call(n=100) == moeq.MOE_ERR_WORKSPACE
    assert call(x=M) == moeq.MOE_ERR_ALIGN
    assert call(H=4092) == moeq.MOE_ERR_UNSUPPORTED


def test_ffn_and_combine_reject_bad_layers(moeq):
    L = moeq.lib()
    good = dict(H=4096, I=1024, E=512, K=4, group=64, bits_routed=4, bits_shared=4, experts=A, shared=A, router_w=A,
                shared_gate_w=None)
    n = moeq.moe_workspace_bytes(1, 4, 4096, 1024, 512)

    def ffn(**kw):
        s = moeq.moe_layer_q(**dict(good, **kw))
        return L.moe_expert_ffn_q(ctypes.byref(s), A, 1, A, A, A, n, None)
    assert ffn(bits_routed=5) == moeq.MOE_ERR_UNSUPPORTED
    assert ffn(bits_routed=3, group=32) == moeq.MOE_ERR_UNSUPPORTED
    assert ffn(group=16) == moeq.MOE_ERR_UNSUPPORTED
    assert ffn(I=1000) == moeq.MOE_ERR_UNSUPPORTED
    assert ffn(K=0) == moeq.MOE_ERR_INVALID_ARG
    assert ffn(K=9) == moeq.MOE_ERR_INVALID_ARG
    assert ffn(experts=None) == moeq.MOE_ERR_INVALID_ARG
    assert ffn(shared=M) == moeq.MOE_ERR_ALIGN
    assert L.moe_expert_ffn_q(None, A, 1, A, A, A, n, None) == moeq.MOE_ERR_INVALID_ARG
    s = moeq.moe_layer_q(**good)
    assert L.moe_expert_ffn_q(ctypes.byref(s), A, 1, A, A, None, n, None) == moeq.MOE_ERR_WORKSPACE
    assert L.moe_expert_ffn_q(ctypes.byref(s), A, 1, A, A, A, 64, None) == moeq.MOE_ERR_WORKSPACE
    assert L.moe_combine_residual(ctypes.byref(s), A, A, A, None, 1, A, None, -1.0, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_combine_residual(ctypes.byref(s), A, A, M, None, 1, A, None, 1e-6, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_combine_residual(ctypes.byref(s), None, A, A, None, 1, A, None, 1e-6, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_get_device_error(None, None) == moeq.MOE_ERR_WORKSPACE
    assert L.moe_workspace_init(None, 0, None) == moeq.MOE_ERR_WORKSPACE


def test_router_rejects_more_experts_than_the_selection_holds(moeq):
    """The router's selection keeps 32 logits per lane of a warp: E > 1024
    is refused on the host instead of silently never picking experts >= 1024."""
    L = moeq.lib()
    n = moeq.moe_workspace_bytes(1, 4, 4096, 1024, 2048)
    assert L.moe_router_topk(A, A, 1, 4096, 2048, 4, 0, None, A, A, None, A, n, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_router_topk(A, A, 1, 4096, 1025, 4, 0, None, A, A, None, A, n, None) == moeq.MOE_ERR_UNSUPPORTED


def test_rmsnorm_and_debug_hook_reject_bad_arguments(moeq):
    L = moeq.lib()
    assert L.moe_rmsnorm(None, None, 1, 4096, 1e-6, A, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(A, None, 1, 4096, 1e-6, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(A, None, 0, 4096, 1e-6, A, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(A, None, 1, 4096, -1.0, A, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(A, None, 1, 4092, 1e-6, A, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_rmsnorm(M, None, 1, 4096, 1e-6, A, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_rmsnorm(A, M, 1, 4096, 1e-6, A, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_workspace_debug(None, 4096, 1000, 1, None) == moeq.MOE_ERR_WORKSPACE
    assert L.moe_workspace_debug(A, 100, 1000, 1, None) == moeq.MOE_ERR_WORKSPACE
    assert L.moe_workspace_debug(M, 4096, 1000, 1, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_workspace_debug(A, 4096, 1000, -1, None) == moeq.MOE_ERR_INVALID_ARG


def test_static_call_checks_arguments_before_its_size(moeq):
    """Every argument error of the static-scratch call returns before the
    scratch-size test (and before anything is queued)."""
    L = moeq.lib()
    good = dict(H=4096, I=1024, E=512, K=4, group=64, bits_routed=4, bits_shared=4, experts=A, shared=A, router_w=A,
                shared_gate_w=None)
    s = moeq.moe_layer_q(**dict(good, K=9))
    assert L.moe_expert_ffn_q_static(ctypes.byref(s), A, 1, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    s = moeq.moe_layer_q(**good)
    assert L.moe_expert_ffn_q_static(ctypes.byref(s), None, 1, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn_q_static(ctypes.byref(s), M, 1, A, A, None, None) == moeq.MOE_ERR_ALIGN
    # a batch too large for the scratch, with a bad pointer: the pointer is reported
    assert L.moe_expert_ffn_q_static(ctypes.byref(s), M, 64, A, A, None, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_expert_ffn_q_static(ctypes.byref(s), A, 64, A, A, None, None) == moeq.MOE_ERR_WORKSPACE
    assert L.moe_expert_ffn_q_static(ctypes.byref(s), A, 35, A, A, None, None) == moeq.MOE_ERR_WORKSPACE


def test_quantize_rejects_bad_arguments(moeq):
    L = moeq.lib()
    assert L.moe_quantize(None, 0, 4, 64, 4, 64, A, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_quantize(A, 2, 4, 64, 4, 64, A, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_quantize(A, 0, -1, 64, 4, 64, A, A, A, None, None) == moeq.MOE_ERR_INVALID_ARG
    assert L.moe_quantize(A, 0, 4, 64, 5, 64, A, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_quantize(A, 0, 4, 96, 4, 64, A, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_quantize(A, 0, 4, 64, 4, 48, A, A, A, None, None) == moeq.MOE_ERR_UNSUPPORTED
    assert L.moe_quantize(M, 0, 4, 64, 4, 64, A, A, A, None, None) == moeq.MOE_ERR_ALIGN
    assert L.moe_quantize(A, 0, 0, 64, 4, 64, A, A, A, None, None) == moeq.MOE_OK  # nothing to do
