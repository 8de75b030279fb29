"""GPU parity of the HARP block builder (harp_blocks, through the C ABI) and of
the HARP transform it feeds into butterfly_apply, against oracle.harp.

Blocks are compared entry by entry (fp32 Gauss-Jordan against the float64
solve: within 2e-6 absolute, the entries of an orthogonal matrix being at most
1 in magnitude); transforms by the fp32 relative-L2 tolerance."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import butterfly as ob
from oracle import hadamard as oh
from oracle import harp as oha
from tests._parity import assert_close, host, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu

BLOCK_ABS = 2e-6

SCHEDULES = [(4096, (16, 16, 16)), (5120, (8, 8, 8, 5, 2)), (14336, (7, 16, 16, 8)), (360, (3, 1, 2, 4, 5, 3))]


def stage_blocks(w, radices, int8, signs=None):
    """Device blocks of every stage; the signs are folded into stage 0."""
    out = []
    for t, b in enumerate(radices):
        mixer = w["base_mixers"].get(b)
        mx = None if mixer is None else to_gpu_f32(mixer)
        s = signs if t == 0 else None
        if b == 1:
            out.append(hit.harp_blocks(None, 1, groups=int(np.prod(radices)), signs=s))
        elif int8:
            q, sc = oha.theta_to_int8(w["thetas"][t])
            out.append(hit.harp_blocks(torch.from_numpy(q).cuda(), b, mixer=mx, signs=s, theta_scale=float(sc)))
        else:
            out.append(hit.harp_blocks(to_gpu_f32(w["thetas"][t]), b, mixer=mx, signs=s))
    return out


def oracle_thetas(w, int8):
    return [oha.theta_from_int8(*oha.theta_to_int8(t)) if int8 else t for t in w["thetas"]]


@pytest.mark.parametrize("d,radices", SCHEDULES)
@pytest.mark.parametrize("int8", [False, True])
def test_blocks_match_oracle(d, radices, int8):
    w = synth.harp_rotation(rows=8, d=d, radices=radices)
    got = stage_blocks(w, radices, int8)
    torch.cuda.synchronize()
    want = oha.blocks(oracle_thetas(w, int8), radices, w["base_mixers"])
    for t, (g, ref) in enumerate(zip(got, want)):
        err = float(np.abs(host(g) - ref).max())
        assert err <= BLOCK_ABS, f"stage {t} (b={radices[t]}): max abs error {err:.2e}"


@pytest.mark.parametrize("d,radices", SCHEDULES[:3])
def test_harp_transform_and_inverse(d, radices):
    """y = R(theta) diag(s) x with the signs folded into stage 0, and the
    inverse diag(s) R(theta)^T y through transpose = 1."""
    w = synth.harp_rotation(rows=64, d=d, radices=radices)
    s = to_gpu_i8(w["signs"])
    blocks = stage_blocks(w, radices, False, signs=s)
    y = hit.butterfly_apply(to_gpu_f32(w["x"]), radices, blocks)
    xr = hit.butterfly_apply(y, radices, blocks, transpose=True)
    torch.cuda.synchronize()
    th = oracle_thetas(w, False)
    ref = oha.forward(w["x"], w["signs"], radices, th, w["base_mixers"])
    assert_close(host(y), ref, torch.float32, "HARP forward")
    assert_close(host(xr), oha.inverse(ref, w["signs"], radices, th, w["base_mixers"]), torch.float32, "HARP inverse")
    assert_close(host(xr), w["x"], torch.float32, "round trip")


def test_zero_parameters_are_the_rht():
    """theta = 0: every block is exactly fp32(H_b / sqrt b) (sign-folded in
    stage 0), and the transform equals rht_forward and the oracle's RHT."""
    radices = (16, 16, 16)
    w = synth.harp_rotation(rows=32, d=4096, radices=radices)
    s = to_gpu_i8(w["signs"])
    zero = [to_gpu_f32(np.zeros_like(t)) for t in w["thetas"]]
    blocks = [hit.harp_blocks(z, 16, signs=s if t == 0 else None) for t, z in enumerate(zero)]
    y = hit.butterfly_apply(to_gpu_f32(w["x"]), radices, blocks)
    z = hit.rht_forward(to_gpu_f32(w["x"]), s)
    torch.cuda.synchronize()
    h = np.float32(0.25) * oh.sylvester(16).astype(np.float32)
    for t, blk in enumerate(blocks):
        ref = np.broadcast_to(h, (256, 16, 16)).copy()
        if t == 0:  # column k of block c reads position k * 256 + c
            ref = ref * w["signs"].reshape(16, 256).T[:, None, :].astype(np.float32)
        assert np.array_equal(blk.cpu().numpy(), ref), f"stage {t}"
    assert_close(host(y), oh.rht_rows(w["x"], w["signs"]), torch.float32, "theta = 0 vs oracle RHT")
    assert_close(host(y), host(z), torch.float32, "theta = 0 vs rht_forward")


def test_int8_parameters_feed_the_full_rotation():
    """int8-stored parameters (per-stage absmax scale) through the device
    builder and butterfly_apply, against the oracle on the dequantized
    parameters, on the two-sided butterfly row schedule (7, 16, 16, 8)."""
    radices = (7, 16, 16, 8)
    w = synth.harp_rotation(rows=16, d=14336, radices=radices)
    blocks = stage_blocks(w, radices, True, signs=to_gpu_i8(w["signs"]))
    y = hit.butterfly_apply(to_gpu_f32(w["x"]), radices, blocks)
    torch.cuda.synchronize()
    ref = oha.forward(w["x"], w["signs"], radices, oracle_thetas(w, True), w["base_mixers"])
    assert_close(host(y), ref, torch.float32, "int8 HARP forward")
