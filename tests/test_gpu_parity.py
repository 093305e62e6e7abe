"""GPU parity: every call of libmoeq.so against the oracle, through the C ABI.

Bars: packed bytes and router indices bit-exact; router weights within 1e-5;
expert and layer outputs within max|err| <= 2e-3 * ||y_oracle||_inf; combine
within 1e-6 relative. Router tests run on tokens whose oracle ranking is
decided by more than twice the a-priori fp32 error bound of the GPU logits
(tests/harness.py::logit_bound); the indices are then compared exactly.
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
from oracle import layer as ref_layer  # noqa: E402
from oracle import oracle as ref  # noqa: E402

FFN_TOL = 2e-3
W_TOL = 1e-5

_layers = {}


def get_layer(name, layer=0, shared_gate=False, **over):
    w = synth.WORKLOADS[name].with_(**over) if over else synth.WORKLOADS[name]
    key = (w, layer, shared_gate)
    if key not in _layers:
        if len(_layers) >= 2:  # keep at most two multi-GB arenas alive
            _layers.clear()
            torch.cuda.empty_cache()
        _layers[key] = hz.build_layer(w, layer, shared_gate)
    return w, _layers[key]


def run_layer(w, L, x, forced=None, renorm=False, resid=None, eps=None):
    B = x.shape[0]
    ws = moeq.Workspace(B, w.K, w.H, w.I, w.E)
    out = L.alloc_outputs(B)
    fi = None if forced is None else torch.as_tensor(np.ascontiguousarray(forced, np.int32), device="cuda")
    L.forward(x, ws, out, resid_in=resid, renorm=renorm, forced_idx=fi, eps=eps)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    return out


def oracle_token(w, layer, x_bits, forced=None, renorm=False, resid=None, shared_gate_bits=None, eps=None):
    experts = hz.oracle_experts(w, layer)
    return ref_layer.layer_token(w.H, w.I, w.E, w.K, w.group, x_bits, synth.router_host(w, layer), experts,
                                 experts(w.E), renorm=renorm, forced=forced, resid=resid,
                                 shared_gate_w=shared_gate_bits, eps=eps)


# ---- generator: the device copy writes the host copy's bytes --------------

def test_device_generator_matches_host():
    w = synth.WORKLOADS["tiny"]
    for (layer, e, m) in ((0, 0, synth.GATE), (3, 8, synth.DOWN), (1, 5, synth.UP)):
        rows, cols = synth.matrix_shape(w, m)
        c = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
        s = torch.empty(rows * cols // w.group, dtype=torch.bfloat16, device="cuda")
        b = torch.empty_like(s)
        synth.fill_matrix_dev(w, layer, e, m, c.data_ptr(), s.data_ptr(), b.data_ptr())
        torch.cuda.synchronize()
        assert (c.cpu().numpy().reshape(rows, cols) == synth.codes_host(w, layer, e, m)).all()
        assert (hz.bf16_bits(s).reshape(rows, -1) == synth.scale_host(w, layer, e, m)).all()
        assert (hz.bf16_bits(b).reshape(rows, -1) == synth.bias_host(w, layer, e, m)).all()
    x = hz.x_device(w, 7, 3)
    assert (hz.bf16_bits(x) == synth.x_host(w, 7, 3)).all()


# ---- A0 pack: byte-exact -----------------------------------------------------

@pytest.mark.parametrize("rows,cols,bits,group", [(1, 32, 4, 32), (5, 64, 2, 32), (37, 320, 4, 64), (129, 256, 2, 64),
                                                  (3, 512, 4, 128), (1024, 4096, 4, 64), (4096, 1024, 2, 64),
                                                  (5, 128, 3, 64), (3, 384, 3, 128), (7, 256, 3, 32),
                                                  (1024, 4096, 3, 64)])
def test_pack_byte_exact(rows, cols, bits, group):
    rng = np.random.default_rng(rows * 7 + cols + bits)
    codes = rng.integers(0, 1 << bits, size=(rows, cols), dtype=np.uint8)
    scale = rng.integers(0, 1 << 16, size=(rows, cols // group), dtype=np.uint16)
    bias = rng.integers(0, 1 << 16, size=(rows, cols // group), dtype=np.uint16)
    dc = torch.from_numpy(codes).cuda()
    ds = torch.from_numpy(scale.view(np.int16)).cuda()
    db = torch.from_numpy(bias.view(np.int16)).cuda()
    packed = torch.full((rows, cols * bits // 8), 0xAB, dtype=torch.uint8, device="cuda")
    sb = torch.full((rows, cols // group, 2), 0x5A5A, dtype=torch.int16, device="cuda")
    ws = moeq.Workspace(1, 1, 32, 32, 1)
    moeq.moe_pack_q(dc, ds, db, rows, cols, bits, group, packed, sb, ws.buf)
    torch.cuda.synchronize()
    rp, rsb = ref.pack(codes, scale, bias, bits, group)
    assert (packed.cpu().numpy() == rp).all()
    assert (sb.cpu().numpy().view(np.uint16) == rsb).all()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK


def test_pack_flags_out_of_range_code():
    rows, cols, bits, group = 4, 64, 4, 32
    codes = np.zeros((rows, cols), np.uint8)
    codes[2, 5] = 16
    ws = moeq.Workspace(1, 1, 32, 32, 1)
    packed = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    sb = torch.empty((rows, 2, 2), dtype=torch.int16, device="cuda")
    z = torch.zeros((rows, 2), dtype=torch.int16, device="cuda")
    moeq.moe_pack_q(torch.from_numpy(codes).cuda(), z, z, rows, cols, bits, group, packed, sb, ws.buf)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_RANGE
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK  # read clears it


def decode_tiles(region, ntiles, C, bits, group):
    """Codes [ntiles, 16, C] and (scale, bias) [ntiles, 16, C/group, 2] of a
    run of record tiles, read back as the header documents them: per tile and
    group a block of 32 lanes x (group/32 k-steps) of lane bytes, then eight
    (row g, row g+8) pairs of bf16 (scale, bias); lane 4*g + t of k-step j
    holds inputs 32j + 8t .. 32j + 8t + 7 of the group for local rows g and
    g + 8."""
    ks, ng = group // 32, C // group
    wb = {4: 8, 3: 6, 2: 4}[bits]
    cb = 32 * ks * wb
    blk = region[:ntiles * ng * (cb + 64)].reshape(ntiles, ng, cb + 64)
    words = np.ascontiguousarray(blk[:, :, :cb]).view("<u4")
    if bits == 4:
        # [T, g, gid, t, j, h] words; nibble i = input 8t + i of local row gid + 8h
        w = words.reshape(ntiles, ng, 8, 4, ks, 2)
        v = (w[..., None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF      # [T, g, gid, t, j, h, i]
        v = v.transpose(0, 5, 2, 1, 4, 3, 6)                                   # [T, h, gid, g, j, t, i]
    elif bits == 3:
        # a 2-bit plane (bits 8i + 2s, s = 2*odd + h, of k-step j's word), then
        # the third bits (bit 8i + 4*(j & 1) + s of word j // 2)
        lo = words[:, :, :32 * ks].reshape(ntiles, ng, 8, 4, ks)
        hw = words[:, :, 32 * ks:].reshape(ntiles, ng, 8, 4, ks // 2)
        hj = np.repeat(hw, 2, axis=-1) >> (4 * (np.arange(ks, dtype=np.uint32) % 2))  # [T, g, gid, t, j]
        sh = 2 * np.arange(16, dtype=np.uint32)                                         # 8i + 2s for the 16 (i, s)
        lo2 = (lo[..., None] >> sh) & 0x3
        hi1 = (hj[..., None] >> (sh // 2 + 4 * (sh // 8))) & 0x1  # 8i + s from 8i + 2s
        v = (lo2 | (hi1 << 2)).reshape(ntiles, ng, 8, 4, ks, 4, 2, 2)                   # [T, g, gid, t, j, i, odd, h]
        v = v.transpose(0, 7, 2, 1, 4, 3, 5, 6)
    else:
        # one word: bits 8i + 4*odd + 2h hold input 8t + 2i + odd of local row gid + 8h
        w = words.reshape(ntiles, ng, 8, 4, ks)
        v = (w[..., None] >> (2 * np.arange(16, dtype=np.uint32))) & 0x3     # position 4i + 2*odd + h
        v = v.reshape(ntiles, ng, 8, 4, ks, 4, 2, 2)                          # [T, g, gid, t, j, i, odd, h]
        v = v.transpose(0, 7, 2, 1, 4, 3, 5, 6)                                # [T, h, gid, g, j, t, i, odd]
    codes = v.reshape(ntiles, 16, C).astype(np.uint8)
    sb = np.ascontiguousarray(blk[:, :, cb:]).view(np.uint16).reshape(ntiles, ng, 8, 2, 2)  # [T, g, gid, h, 2]
    sb = sb.transpose(0, 3, 2, 1, 4).reshape(ntiles, 16, ng, 2)
    return codes, sb


def record_rows(rec, lay, H, I, bits, group):
    """Gate, up and down as (codes [rows, cols], (scale, bias) [rows, cols/group, 2])
    read back out of one record (numpy u8) with the layout moe_expert_layout gives."""
    U, down_off, D, rows_per_tile, blk, gu_tiles = lay
    assert rows_per_tile == 16 and gu_tiles == I // 8
    gc, gsb = decode_tiles(rec[:gu_tiles * U], gu_tiles, H, bits, group)
    dc, dsb = decode_tiles(rec[down_off:down_off + (H // 16) * D], H // 16, I, bits, group)
    gate = (gc[:, :8].reshape(I, H), gsb[:, :8].reshape(I, H // group, 2))
    up = (gc[:, 8:].reshape(I, H), gsb[:, 8:].reshape(I, H // group, 2))
    down = (dc.reshape(H, I), dsb.reshape(H, I // group, 2))
    return gate, up, down


@pytest.mark.parametrize("name,over", [("tiny", {}), ("tiny", dict(bits_routed=2, bits_shared=2, group=64)),
                                       ("tiny", dict(bits_routed=2, bits_shared=4, group=128)),
                                       ("tiny", dict(bits_routed=3, bits_shared=3, group=64)),
                                       ("tiny", dict(bits_routed=3, bits_shared=4, group=128))])
def test_packed_arena_matches_generator(name, over):
    w = synth.WORKLOADS[name].with_(**over)
    L = hz.build_layer(w, 0)
    torch.cuda.synchronize()
    arena = L.experts.cpu().numpy()
    shared = L.shared.cpu().numpy()
    for e in (0, w.E - 1, w.E):
        rec = shared if e == w.E else arena[e * L.rec_r:(e + 1) * L.rec_r]
        lay = L.lay_s if e == w.E else L.lay_r
        got = record_rows(rec, lay, w.H, w.I, w.bits_of(e), w.group)
        for m, (codes, scale, bias) in enumerate(synth.expert_host(w, 0, e)):
            assert (got[m][0] == codes).all(), (e, m)
            assert (got[m][1][..., 0] == scale).all(), (e, m)
            assert (got[m][1][..., 1] == bias).all(), (e, m)


# ---- A1+A2 router ------------------------------------------------------------

@pytest.mark.parametrize("name,B,renorm", [("tiny", 1, False), ("tiny", 3, True), ("layer4", 1, False),
                                           ("layer4", 5, True), ("layer4", 32, False)])
def test_router_topk(name, B, renorm):
    """Router indices bit-exact on every token: the tokens are the first ones
    whose oracle ranking is decided by more than twice the a-priori fp32
    error bound of the GPU logits (tokens with a near tie are skipped and
    reported, never compared loosely)."""
    w, L = get_layer(name)
    toks, skipped = hz.decided_tokens(w, 0, B, 100, ref.router_logits)
    x = hz.x_tokens_device(w, toks)
    ws = moeq.Workspace(B, w.K, w.H, w.I, w.E)
    idx = torch.empty((B, w.K), dtype=torch.int32, device="cuda")
    wt = torch.empty((B, w.K), dtype=torch.float32, device="cuda")
    lg = torch.empty((B, w.E), dtype=torch.float32, device="cuda")
    moeq.moe_router_topk(x, L.router_w, B, w.H, w.E, w.K, renorm, None, idx, wt, lg, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    wr = synth.router_host(w, 0)
    for b, t in enumerate(toks):
        xb = synth.x_host(w, t)[0]
        rl = ref.router_logits(xb, wr)
        bound = hz.logit_bound(xb, wr)
        assert (np.abs(lg[b].cpu().numpy() - rl) <= bound).all()
        ri, rw = ref.topk(rl, w.K, renorm=renorm)
        assert list(idx[b].cpu().numpy()) == list(ri), (t, idx[b].tolist(), list(ri))
        assert np.abs(wt[b].cpu().numpy() - rw).max() <= W_TOL
    print("near-tie tokens skipped:", skipped)


def test_router_forced_and_bad_index():
    w, L = get_layer("tiny")
    B = 2
    x = hz.x_device(w, 3, B)
    ws = moeq.Workspace(B, w.K, w.H, w.I, w.E)
    forced = torch.tensor([[3, 1], [0, 7]], dtype=torch.int32, device="cuda")
    idx = torch.empty((B, w.K), dtype=torch.int32, device="cuda")
    wt = torch.empty((B, w.K), dtype=torch.float32, device="cuda")
    moeq.moe_router_topk(x, L.router_w, B, w.H, w.E, w.K, False, forced, idx, wt, None, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert (idx == forced).all()
    wr = synth.router_host(w, 0)
    xb = synth.x_host(w, 3, B)
    for b in range(B):
        _, rw = ref.topk(ref.router_logits(xb[b], wr), w.K, forced=forced[b].cpu().numpy())
        assert np.abs(wt[b].cpu().numpy() - rw).max() <= W_TOL
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    bad = torch.tensor([[3, 8], [0, -1]], dtype=torch.int32, device="cuda")
    moeq.moe_router_topk(x, L.router_w, B, w.H, w.E, w.K, False, bad, idx, wt, None, ws.buf, ws.nbytes)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_INDEX


# ---- A3..A5 expert FFN ---------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "layer4", "layer2", "layer3"])
def test_expert_ffn(name):
    w, L = get_layer(name)
    B = 2
    x = hz.x_device(w, 11, B)
    rng = np.random.default_rng(5)
    idx_np = np.stack([rng.choice(w.E, size=w.K, replace=False) for _ in range(B)]).astype(np.int32)
    idx = torch.from_numpy(idx_np).cuda()
    ws = moeq.Workspace(B, w.K, w.H, w.I, w.E)
    y = torch.empty((B, w.K + 1, w.H), dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, B, idx, y, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    experts = hz.oracle_experts(w, 0)
    xb = synth.x_host(w, 11, B)
    yg = y.cpu().numpy()
    for b in range(B):
        xd = hz.bf16_to_f64(xb[b])
        for k, e in enumerate(list(idx_np[b]) + [w.E]):
            g, u, d = experts(int(e))
            yr = ref.expert_ffn(w.H, w.I, w.group, g, u, d, xd)
            assert hz.max_rel_err(yg[b, k], yr) <= FFN_TOL, (b, k, e, hz.max_rel_err(yg[b, k], yr))


@pytest.mark.parametrize("bits_routed", [4, 2])
def test_expert_ffn_one_token_in_rounds(bits_routed):
    """One token through moe_expert_ffn_q at H=4096, I=8192, K=2: a CTA's share
    is about 21 gate/up tiles (36,864 B each, five fit shared memory) and 6
    down tiles (73,728 B each, two fit), so both kernels work in rounds."""
    w = synth.WORKLOADS["layer4"].with_(name="rounds", I=8192, E=8, K=2, bits_routed=bits_routed)
    L = hz.build_layer(w, 0)
    x = hz.x_device(w, 21, 1)
    idx_np = np.array([[5, 2]], dtype=np.int32)
    idx = torch.from_numpy(idx_np).cuda()
    ws = moeq.Workspace(1, w.K, w.H, w.I, w.E)
    y = torch.empty((1, w.K + 1, w.H), dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, 1, idx, y, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    experts = hz.oracle_experts(w, 0)
    xd = hz.bf16_to_f64(synth.x_host(w, 21, 1)[0])
    yg = y.cpu().numpy()
    for k, e in enumerate(list(idx_np[0]) + [w.E]):
        g, u, d = experts(int(e))
        yr = ref.expert_ffn(w.H, w.I, w.group, g, u, d, xd)
        assert hz.max_rel_err(yg[0, k], yr) <= FFN_TOL, (k, e, hz.max_rel_err(yg[0, k], yr))
    del L
    torch.cuda.empty_cache()


def test_expert_ffn_bad_index_zeroes_slot():
    w, L = get_layer("tiny")
    x = hz.x_device(w, 1, 1)
    idx = torch.tensor([[1, 99]], dtype=torch.int32, device="cuda")
    ws = moeq.Workspace(1, w.K, w.H, w.I, w.E)
    y = torch.full((1, w.K + 1, w.H), 7.0, dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, 1, idx, y, ws.buf, ws.nbytes)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_INDEX
    assert (y[0, 1] == 0).all() and (y[0, 0] != 0).any() and (y[0, 2] != 0).any()


def test_grouped_batch_repeats_and_bad_index():
    """A full batch whose picks repeat one expert (so that expert has more
    entries than one work item holds) plus one index out of range."""
    w, L = get_layer("tiny")
    B = moeq.MOEQ_MAX_B
    x = hz.x_device(w, 77, B)
    idx_np = np.full((B, w.K), 3, dtype=np.int32)
    idx_np[:, -1] = (np.arange(B) % w.E).astype(np.int32)
    idx_np[5, 1] = 99
    idx = torch.from_numpy(idx_np).cuda()
    ws = moeq.Workspace(B, w.K, w.H, w.I, w.E)
    y = torch.full((B, w.K + 1, w.H), 7.0, dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, B, idx, y, ws.buf, ws.nbytes)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_INDEX
    yg = y.cpu().numpy()
    assert (yg[5, 1] == 0).all()
    experts = hz.oracle_experts(w, 0)
    xb = synth.x_host(w, 77, B)
    for b in (0, 5, 31, B - 1):
        xd = hz.bf16_to_f64(xb[b])
        for k, e in enumerate(list(idx_np[b]) + [w.E]):
            if e >= w.E and k < w.K:
                continue
            g, u, d = experts(int(e))
            yr = ref.expert_ffn(w.H, w.I, w.group, g, u, d, xd)
            assert hz.max_rel_err(yg[b, k], yr) <= FFN_TOL, (b, k, e)


# ---- A6 combine ------------------------------------------------------------------

@pytest.mark.parametrize("with_gate,with_resid", [(False, False), (True, True)])
def test_combine_residual(with_gate, with_resid):
    w, L = get_layer("tiny", shared_gate=with_gate)
    B = 3
    rng = np.random.default_rng(9)
    y = torch.from_numpy(rng.normal(size=(B, w.K + 1, w.H)).astype(np.float32)).cuda()
    wt = torch.from_numpy(rng.uniform(size=(B, w.K)).astype(np.float32)).cuda()
    x = hz.x_device(w, 40, B)
    resid = torch.from_numpy(synth.resid_host(w, 40, B)).cuda() if with_resid else None
    out = torch.empty((B, w.H), dtype=torch.float32, device="cuda")
    xn = torch.empty((B, w.H), dtype=torch.bfloat16, device="cuda")
    moeq.moe_combine_residual(L.struct, y, wt, x, resid, B, out, xn, 1e-6)
    torch.cuda.synchronize()
    xb = synth.x_host(w, 40, B)
    gw = synth.shared_gate_host(w, 0) if with_gate else None
    for b in range(B):
        gamma = ref.shared_gate(gw, xb[b]) if with_gate else 1.0
        r = resid[b].cpu().numpy().astype(np.float64) if with_resid else hz.bf16_to_f64(xb[b])
        ro = ref.combine(y[b].cpu().numpy().astype(np.float64), wt[b].cpu().numpy().astype(np.float64), gamma, r)
        assert hz.max_rel_err(out[b].cpu().numpy(), ro) <= 1e-6
        rn = ref.rmsnorm(ro, 1e-6)
        xg = hz.bf16_to_f64(hz.bf16_bits(xn[b]))
        # one bf16 rounding apart at most
        assert (np.abs(xg - rn) <= np.abs(rn) * 2.0 ** -8 + 1e-30).all()


@pytest.mark.parametrize("H,with_norm", [(4096, True), (4096, False), (16448, True)])
def test_combine_residual_shapes(H, with_norm):
    """The combine at the layer width (one row per thread of each cluster
    CTA), without the normalised copy, and at a width where a thread owns
    several rows (the partial sums of squares still meet across the cluster)."""
    K, B = 4, 2
    L = moeq.moe_layer_q(H=H, I=1024, E=64, K=K, group=64, bits_routed=4, bits_shared=4, experts=0x10000,
                         shared=0x10000, router_w=0x10000, shared_gate_w=None)
    rng = np.random.default_rng(H + with_norm)
    y = torch.from_numpy(rng.normal(size=(B, K + 1, H)).astype(np.float32)).cuda()
    wt = torch.from_numpy(rng.uniform(size=(B, K)).astype(np.float32)).cuda()
    x = torch.from_numpy(rng.normal(size=(B, H)).astype(np.float32)).to(torch.bfloat16).cuda()
    resid = torch.from_numpy(rng.normal(size=(B, H)).astype(np.float32)).cuda()
    out = torch.empty((B, H), dtype=torch.float32, device="cuda")
    xn = torch.empty((B, H), dtype=torch.bfloat16, device="cuda") if with_norm else None
    moeq.moe_combine_residual(L, y, wt, x, resid, B, out, xn, 1e-6)
    torch.cuda.synchronize()
    for b in range(B):
        yb, wb, rb = (t[b].cpu().numpy().astype(np.float64) for t in (y, wt, resid))
        ro = ref.combine(yb, wb, 1.0, rb)
        assert hz.max_rel_err(out[b].cpu().numpy(), ro) <= 1e-6
        if with_norm:
            rn = ref.rmsnorm(ro, 1e-6)
            xg = hz.bf16_to_f64(hz.bf16_bits(xn[b]))
            # one bf16 rounding, plus the fp32 error of r itself carried
            # through 1/RMS: r = r_in + sum_k w_k y_k in fp32 is off by up to
            # (K + 2) * 2^-23 * (|r_in| + sum_k |w_k y_k|) per element, which
            # matters where the terms cancel
            inv = np.abs(rn).sum() / np.abs(ro).sum()
            mag = np.abs(rb) + (np.abs(wb[:, None] * yb[:K]).sum(axis=0)) + np.abs(yb[K])
            assert (np.abs(xg - rn) <= np.abs(rn) * 2.0 ** -8 + inv * (K + 2) * 2.0 ** -23 * mag + 1e-30).all()


# ---- A1..A6 whole layer -----------------------------------------------------------

@pytest.mark.parametrize("name,B", [("tiny", 1), ("tiny", 4), ("layer4", 1), ("layer2", 1), ("layer4", 3),
                                    ("layer3", 1), ("layer3", 4)])
def test_layer_end_to_end(name, B):
    """The three per-token calls against the oracle layer: indices exact on
    tokens whose ranking is decided (near-tie tokens are skipped, reported),
    weights, every expert slot and the residual output within the bars."""
    w, L = get_layer(name)
    toks, skipped = hz.decided_tokens(w, 0, B, 500, ref.router_logits)
    x = hz.x_tokens_device(w, toks)
    out = run_layer(w, L, x, eps=1e-6)
    for b, t in enumerate(toks):
        ro = oracle_token(w, 0, synth.x_host(w, t)[0], eps=1e-6)
        assert list(out["idx"][b].cpu().numpy()) == list(ro["idx"]), (t, out["idx"][b].tolist(), list(ro["idx"]))
        assert np.abs(out["w"][b].cpu().numpy() - ro["w"]).max() <= W_TOL
        yg = out["y"][b].cpu().numpy()
        for k in range(w.K + 1):
            assert hz.max_rel_err(yg[k], ro["y"][k]) <= FFN_TOL
        assert hz.max_rel_err(out["resid"][b].cpu().numpy(), ro["out"]) <= FFN_TOL
    print("near-tie tokens skipped:", skipped)


@pytest.mark.parametrize("over,B", [(dict(E=1024, K=8, group=128), 1), (dict(E=1024, K=8, group=128), 5),
                                    (dict(bits_routed=2, bits_shared=2), 1), (dict(bits_routed=3, bits_shared=3,
                                                                                   group=128), 3)],
                         ids=["E1024-K8-g128-B1", "E1024-K8-g128-B5", "2bit-both-B1", "3bit-both-g128-B3"])
def test_layer_end_to_end_other_shapes(over, B):
    """The three per-token calls at the most experts and picks (E 1024, K 8),
    at group 128 and with the shared expert at the routed width, for one token
    and for a grouped batch: indices, weights, every slot and the residual."""
    w, L = get_layer("layer4", **over)
    toks, skipped = hz.decided_tokens(w, 0, B, 500, ref.router_logits)
    x = hz.x_tokens_device(w, toks)
    out = run_layer(w, L, x, eps=1e-6)
    for b, t in enumerate(toks):
        ro = oracle_token(w, 0, synth.x_host(w, t)[0], eps=1e-6)
        assert list(out["idx"][b].cpu().numpy()) == list(ro["idx"]), (t, out["idx"][b].tolist(), list(ro["idx"]))
        assert np.abs(out["w"][b].cpu().numpy() - ro["w"]).max() <= W_TOL
        yg = out["y"][b].cpu().numpy()
        for k in range(w.K + 1):
            assert hz.max_rel_err(yg[k], ro["y"][k]) <= FFN_TOL
        assert hz.max_rel_err(out["resid"][b].cpu().numpy(), ro["out"]) <= FFN_TOL
    print("near-tie tokens skipped:", skipped)


@pytest.mark.parametrize("B", [64, 128])
def test_batched_zipf_larger_batches(B):
    """Batches of 64 and 128 tokens on the layer4 arena (Zipf(1.1) picks, so
    popular experts carry many tokens and the shared expert carries all of
    them): every token's weights, every expert slot and every residual row
    against the oracle (the oracle runs the tokens on a thread pool)."""
    from concurrent.futures import ThreadPoolExecutor
    import os
    w, L = get_layer("batch32")
    routing = synth.zipf_routing(w.E, w.K, B, 1, w.zipf_s, 17 + B)[0]
    x = hz.x_device(w, 3000 + B, B)
    out = run_layer(w, L, x, forced=routing)
    xb = synth.x_host(w, 3000 + B, B)
    yg = out["y"].cpu().numpy()
    wg = out["w"].cpu().numpy()
    rg = out["resid"].cpu().numpy()
    def one(b):
        return b, oracle_token(w, 0, xb[b], forced=routing[b])

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as pool:
        for b, ro in pool.map(one, range(B)):
            assert np.abs(wg[b] - ro["w"]).max() <= W_TOL, b
            for k in range(w.K + 1):
                assert hz.max_rel_err(yg[b, k], ro["y"][k]) <= FFN_TOL, (b, k)
            assert hz.max_rel_err(rg[b], ro["out"]) <= FFN_TOL, b


def test_batched_zipf_routing_layer():
    """The batched workload (32 tokens, forced Zipf(1.1) picks, grouped per
    expert): every token's weights, every expert slot of y and every
    residual row against the oracle."""
    w, L = get_layer("batch32")
    routing = synth.zipf_routing(w.E, w.K, w.B, 1, w.zipf_s, w.seed)[0]
    x = hz.x_device(w, 900, w.B)
    out = run_layer(w, L, x, forced=routing)
    xb = synth.x_host(w, 900, w.B)
    yg = out["y"].cpu().numpy()
    for b in range(w.B):
        ro = oracle_token(w, 0, xb[b], forced=routing[b])
        assert (out["idx"][b].cpu().numpy() == routing[b]).all()
        assert np.abs(out["w"][b].cpu().numpy() - ro["w"]).max() <= W_TOL
        for k in range(w.K + 1):
            assert hz.max_rel_err(yg[b, k], ro["y"][k]) <= FFN_TOL, (b, k)
        assert hz.max_rel_err(out["resid"][b].cpu().numpy(), ro["out"]) <= FFN_TOL


@pytest.mark.parametrize("over", [dict(H=320, I=96, E=5, K=1, group=32), dict(H=512, I=192, E=9, K=8, group=64),
                                  dict(H=512, I=128, E=6, K=3, group=128, bits_routed=2),
                                  dict(H=256, I=64, E=4, K=4, group=32, bits_routed=2, bits_shared=2),
                                  dict(H=384, I=128, E=5, K=2, group=64, bits_routed=3, bits_shared=3),
                                  dict(H=640, I=256, E=7, K=3, group=128, bits_routed=3)])
@pytest.mark.parametrize("B", [1, 3])
def test_ragged_and_edge_shapes(over, B):
    w = synth.WORKLOADS["tiny"].with_(**over)
    L = hz.build_layer(w, 2)
    toks, _ = hz.decided_tokens(w, 2, B, 77, ref.router_logits)
    x = hz.x_tokens_device(w, toks)
    out = run_layer(w, L, x, eps=1e-6)
    for b, t in enumerate(toks):
        ro = oracle_token(w, 2, synth.x_host(w, t)[0], eps=1e-6)
        assert list(out["idx"][b].cpu().numpy()) == list(ro["idx"])
        assert np.abs(out["w"][b].cpu().numpy() - ro["w"]).max() <= W_TOL
        assert hz.max_rel_err(out["resid"][b].cpu().numpy(), ro["out"]) <= FFN_TOL
        for k in range(w.K + 1):
            assert hz.max_rel_err(out["y"][b, k].cpu().numpy(), ro["y"][k]) <= FFN_TOL


# ---- standalone RMS norm -------------------------------------------------------

@pytest.mark.parametrize("B,H,weighted", [(1, 4096, False), (3, 4096, True), (5, 264, True), (64, 512, False)])
def test_rmsnorm(B, H, weighted):
    """moe_rmsnorm against the oracle's weighted RMS norm: every output is the
    oracle's bf16 value or its neighbour (the fp32 product may land on the
    other side of a rounding boundary), and almost all are identical."""
    rng = np.random.default_rng(B * 1000 + H)
    r = (rng.normal(size=(B, H)) * rng.uniform(0.1, 30.0, size=(B, 1))).astype(np.float32)
    wbits = None
    if weighted:
        wbits = (rng.normal(1.0, 0.3, size=H).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    rd = torch.from_numpy(r).cuda()
    wd = torch.from_numpy(wbits.view(np.int16)).cuda() if weighted else None
    xn = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
    moeq.moe_rmsnorm(rd, wd, B, H, 1e-6, xn)
    torch.cuda.synchronize()
    got = hz.bf16_bits(xn).astype(np.int32)
    same = 0
    for b in range(B):
        want = ref.rmsnorm_weighted_bf16(r[b].astype(np.float64), wbits, 1e-6).astype(np.int32)
        sign_ok = ((got[b] ^ want) & 0x8000) == 0
        assert (sign_ok | ((got[b] | want) & 0x7FFF == 0)).all()
        assert (np.abs((got[b] & 0x7FFF) - (want & 0x7FFF)) <= 1).all(), b
        same += int((got[b] == want).sum())
    assert same >= 0.99 * B * H


# ---- quantisation (weights -> codes, scale, bias) -------------------------------

def _weights(rng, rows, cols, group):
    """fp32 weights with groups of every kind the quantiser meets: spread
    normal rows, groups far from zero for their range (the bias rounds away
    from the minimum, so codes clamp), and constant groups (scale 0)."""
    w = rng.normal(size=(rows, cols)) * rng.uniform(0.005, 3.0, size=(rows, 1))
    far = rng.choice([-1.0, 1.0], size=(rows, 1)) * rng.uniform(60.0, 130.0, size=(rows, 1))
    w[1::3] = far[1::3] + rng.uniform(0.0, 1.0, size=w[1::3].shape)
    w[2::5, :group] = 0.375
    return w.astype(np.float32)


@pytest.mark.parametrize("rows,cols,bits,group", [(37, 256, 4, 32), (64, 512, 3, 64), (5, 1024, 2, 128),
                                                  (1024, 4096, 4, 64), (4096, 1024, 3, 64), (3, 384, 3, 128)])
@pytest.mark.parametrize("in_bf16", [False, True])
def test_quantize_bit_exact(rows, cols, bits, group, in_bf16):
    """moe_quantize against the oracle: codes, scale and bias identical bit
    for bit (both decide the codes in binary32)."""
    rng = np.random.default_rng(rows + cols + bits)
    w = _weights(rng, rows, cols, group)
    if in_bf16:
        bits16 = (w.view(np.uint32) >> 16).astype(np.uint16)  # truncate to bf16, then both sides read that
        w = (bits16.astype(np.uint32) << 16).view(np.float32)
        wd = torch.from_numpy(bits16.view(np.int16)).cuda()
    else:
        wd = torch.from_numpy(w).cuda()
    codes = torch.full((rows, cols), 0xEE, dtype=torch.uint8, device="cuda")
    sc = torch.empty((rows, cols // group), dtype=torch.int16, device="cuda")
    bi = torch.empty_like(sc)
    ws = moeq.Workspace(1, 1, 32, 32, 1)
    moeq.moe_quantize(wd, in_bf16, rows, cols, bits, group, codes, sc, bi, ws.buf)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    rc, rs, rb = ref.quantize(w, bits, group)
    assert (codes.cpu().numpy() == rc).all()
    assert (sc.cpu().numpy().view(np.uint16) == rs).all()
    assert (bi.cpu().numpy().view(np.uint16) == rb).all()


def test_quantize_flags_non_finite_group():
    w = np.ones((2, 128), np.float32)
    w[1, 70] = np.inf
    codes = torch.full((2, 128), 9, dtype=torch.uint8, device="cuda")
    sc = torch.full((2, 2), 1, dtype=torch.int16, device="cuda")
    bi = torch.full((2, 2), 1, dtype=torch.int16, device="cuda")
    ws = moeq.Workspace(1, 1, 32, 32, 1)
    moeq.moe_quantize(torch.from_numpy(w).cuda(), False, 2, 128, 4, 64, codes, sc, bi, ws.buf)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_RANGE
    c = codes.cpu().numpy()
    assert (c[1, 64:] == 0).all() and int(sc[1, 1]) == 0 and int(bi[1, 1]) == 0
    assert int(bi[0, 0]) == 0x3F80 and int(sc[1, 0]) == 0  # the other groups as usual (constant 1.0)


@pytest.mark.parametrize("bits,group", [(3, 64), (4, 64), (2, 128), (3, 128)])
def test_quantize_pack_and_run_expert(bits, group):
    """fp32 weights through the whole set-up path on the GPU (moe_quantize,
    then moe_pack_expert) and one token through the resulting 3-matrix
    expert, against the oracle's quantiser and expert FFN on the same
    weights."""
    H, I, E, K = 512, 256, 2, 1
    rng = np.random.default_rng(bits * 100 + group)
    mats = [(rng.normal(size=(I, H)) * 0.05).astype(np.float32), (rng.normal(size=(I, H)) * 0.05).astype(np.float32),
            (rng.normal(size=(H, I)) * 0.05).astype(np.float32)]
    L = moeq.QuantLayer(H, I, E, K, group, bits, bits)
    ws = moeq.Workspace(1, K, H, I, E)
    dev = []
    for m in mats:
        r, c = m.shape
        codes = torch.empty((r, c), dtype=torch.uint8, device="cuda")
        sc = torch.empty((r, c // group), dtype=torch.int16, device="cuda")
        bi = torch.empty_like(sc)
        moeq.moe_quantize(torch.from_numpy(m).cuda(), False, r, c, bits, group, codes, sc, bi, ws.buf)
        dev.append((codes, sc, bi))
    for e in range(E + 1):
        L.pack_expert(e, *dev, ws=ws.buf)
    L.router_w.zero_()
    x_bits = (rng.normal(size=H).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)[None, :]
    idx = torch.tensor([[1]], dtype=torch.int32, device="cuda")
    y = torch.empty((1, K + 1, H), dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, 1, idx, y, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    q = [ref.quantize(m, bits, group) for m in mats]
    yr = ref.expert_ffn(H, I, group, q[0], q[1], q[2], hz.bf16_to_f64(x_bits))
    for k in range(K + 1):
        assert hz.max_rel_err(y[0, k].cpu().numpy(), yr) <= FFN_TOL, k


# ---- the CUDA-core comparison dot of the one-token kernels ---------------------

_FMA_CHECK = r'''
import sys
import numpy as np
import torch
sys.path.insert(0, ".")
from synth import synth
from tests import harness as hz
from oracle import oracle as ref
import quantized_expert_ffn_topk_b200 as moeq
for name in ("layer4", "layer3", "tiny"):
    w = synth.WORKLOADS[name]
    L = hz.build_layer(w, 0)
    x = hz.x_device(w, 31, 1)
    idx_np = np.random.default_rng(3).choice(w.E, size=(1, w.K), replace=False).astype(np.int32)
    ws = moeq.Workspace(1, w.K, w.H, w.I, w.E)
    y = torch.empty((1, w.K + 1, w.H), dtype=torch.float32, device="cuda")
    moeq.moe_expert_ffn_q(L.struct, x, 1, torch.from_numpy(idx_np).cuda(), y, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    experts = hz.oracle_experts(w, 0)
    xd = hz.bf16_to_f64(synth.x_host(w, 31, 1)[0])
    for k, e in enumerate(list(idx_np[0]) + [w.E]):
        g, u, d = experts(int(e))
        err = hz.max_rel_err(y[0, k].cpu().numpy(), ref.expert_ffn(w.H, w.I, w.group, g, u, d, xd))
        assert err <= 2e-3, (name, k, err)
    del L
    torch.cuda.empty_cache()
print("fma dot ok")
'''


def test_expert_ffn_cuda_core_dot():
    """The one-token expert FFN with its dots on the CUDA cores in fp32
    (MOEQ_BATCH1_DOT=fma, read once per process, hence a child process): the
    same parity bar as the tensor-core dot."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FMA_CHECK], cwd=root, capture_output=True, text=True, timeout=900,
                       env=dict(os.environ, MOEQ_BATCH1_DOT="fma"))
    assert r.returncode == 0 and "fma dot ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
