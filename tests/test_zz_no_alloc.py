"""moe_expert_ffn_q_static: the expert FFN call for callers that cannot
allocate device memory (they are handed only their input and output buffers,
or run where cudaMalloc may not be called), so it runs on a scratch array
inside the library instead of a caller workspace.

Its outputs must match moe_expert_ffn_q's on the same inputs, call after call
(the scratch keeps the previous call's contents), within the expert-output
tolerance of the parity tests: max|err| <= 2e-3 * ||y||_inf. This file is
collected last so that a failure here leaves every other test already run.
"""
import numpy as np
import pytest

from synth import synth
from tests import harness as hz

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import quantized_expert_ffn_topk_b200 as moeq  # noqa: E402

FFN_TOL = 2e-3


_layers = {}


def _layer(name):
    if name not in _layers:
        _layers[name] = hz.build_layer(synth.WORKLOADS[name], 0)
    return _layers[name]


def _picks(w, B, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(w.E, size=w.K, replace=False) for _ in range(B)]).astype(np.int32)
    return torch.from_numpy(idx).cuda()


def _with_workspace(L, w, x, B, idx):
    ws = moeq.Workspace(B, w.K, w.H, w.I, w.E)
    y = torch.empty((B, w.K + 1, w.H), dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, B, idx, y, ws.buf, ws.nbytes)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    return y


def _rel(got, want):
    return float((got - want).abs().max() / want.abs().max().clamp_min(1e-30))


@pytest.mark.parametrize("name,B", [("tiny", 3), ("layer4", 2)])
def test_static_scratch_matches_workspace_call(name, B):
    w = synth.WORKLOADS[name]
    L = _layer(name)
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    # two calls in a row on different tokens and picks: the second runs on
    # the scratch the first left behind
    for call, (token, seed) in enumerate([(3, 21), (17, 22)]):
        x = hz.x_device(w, token, B)
        idx = _picks(w, B, seed)
        y = torch.full((B, w.K + 1, w.H), float("nan"), dtype=torch.float32, device="cuda")
        moeq.moe_expert_ffn_q_static(L.struct, x, B, idx, y, err)
        torch.cuda.synchronize()
        assert int(err.item()) == moeq.MOE_OK, call
        want = _with_workspace(L, w, x, B, idx)
        torch.cuda.synchronize()
        assert torch.isfinite(y).all(), call
        assert _rel(y, want) <= FFN_TOL, (call, _rel(y, want))


def test_static_scratch_reports_bad_index_then_clears():
    w = synth.WORKLOADS["tiny"]
    L = _layer("tiny")
    x = hz.x_device(w, 1, 1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((1, w.K + 1, w.H), 7.0, dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q_static(L.struct, x, 1, torch.tensor([[1, 99]], dtype=torch.int32, device="cuda"), y, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moeq.MOE_ERR_INDEX
    assert (y[0, 1] == 0).all() and (y[0, 0] != 0).any()
    # the next call starts from a cleared control block
    idx = torch.tensor([[1, 2]], dtype=torch.int32, device="cuda")
    moeq.moe_expert_ffn_q_static(L.struct, x, 1, idx, y, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moeq.MOE_OK
    assert _rel(y, _with_workspace(L, w, x, 1, idx)) <= FFN_TOL


def test_static_scratch_rejects_shapes_over_its_size():
    w = synth.WORKLOADS["layer4"]
    B = moeq.MOEQ_MAX_B
    assert moeq.moe_workspace_bytes(B, w.K, w.H, w.I, w.E) > moeq.MOEQ_STATIC_SCRATCH_BYTES
    L = _layer("layer4")  # a real arena, so nothing could read outside it
    x = torch.zeros((B, w.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((B, w.K), dtype=torch.int32, device="cuda")
    y = torch.empty((B, w.K + 1, w.H), dtype=torch.float32, device="cuda")
    with pytest.raises(moeq.MoeError) as e:
        moeq.moe_expert_ffn_q_static(L.struct, x, B, idx, y)
    assert e.value.status == moeq.MOE_ERR_WORKSPACE
