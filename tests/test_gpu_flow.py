"""GPU parity of the flow-matching elementwise kernels (SkyReels-V4 digest,
step 4) against the fp64 oracle: the fused noised input / velocity target and
the per-item loss term, bf16 and fp32, ragged item lengths and padded item
strides (the padding must stay untouched).  Tolerances, elementwise: an
output stored in bf16 is the fp32 result rounded once, so it lies within one
bf16 unit in the last place of the oracle's value (2^-8 relative) plus the
fp32 rounding of the interpolation (1e-6 absolute; the target z0 - eps of
bf16 inputs is exact in fp32); fp32 outputs within 1e-5.  The loss, an fp32
sum of the stored values' squared differences, relative 1e-5."""
import numpy as np
import pytest

import oracle as O
from joint_video_audio_rope_b200 import workloads as WL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from joint_video_audio_rope_b200 import build
    build.build()
    from joint_video_audio_rope_b200 import mmdit
    return mmdit


CASES = {
    # a 480p video latent per item (21 x 30 x 52 positions x 16 channels)
    "video_bf16": dict(batch=3, n=21 * 30 * 52 * 16, pad=0, dtype="bf16"),
    # ragged length and a padded stride
    "ragged_bf16": dict(batch=3, n=1001, pad=7, dtype="bf16"),
    "audio_f32": dict(batch=2, n=218 * 128, pad=0, dtype="f32"),
    "ragged_f32": dict(batch=4, n=37, pad=3, dtype="f32"),
    "tiny_bf16": dict(batch=2, n=5, pad=3, dtype="bf16"),
}


def _tensors(c, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    b, n, pad = c["batch"], c["n"], c["pad"]
    arrs = [rng.standard_normal((b, n + pad), dtype=np.float32) for _ in range(3)]
    t = np.linspace(0.0, 1.0, b).astype(np.float32)  # includes both endpoints
    if c["dtype"] == "bf16":
        host = [WL.bf16_bits_to_f32(WL.f32_to_bf16_bits(a)) for a in arrs]
        dev = [torch.from_numpy(WL.f32_to_bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
               for a in arrs]
    else:
        host = arrs
        dev = [torch.from_numpy(a).cuda() for a in arrs]
    return [h.astype(np.float64) for h in host], dev, t


def _f64(x):
    return x.float().cpu().numpy().astype(np.float64)


def _check(got, ref, dtype, what):
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6 if dtype == "bf16" else np.full_like(ref, 1e-5)
    worst = np.argmax(err - bound)
    assert np.all(err <= bound), f"{what}: |err| {err.flat[worst]:.3e} > {bound.flat[worst]:.3e}"


@pytest.mark.parametrize("case", list(CASES))
def test_flow_noise(M, case):
    c = CASES[case]
    (z0, eps, _), (dz0, deps, _), t = _tensors(c, 11)
    n = c["n"]
    zt = torch.full_like(dz0, 3.0)
    u = torch.full_like(dz0, 3.0)
    M.flow_noise(dz0[:, :n], deps[:, :n], torch.from_numpy(t).cuda(), zt[:, :n], u[:, :n])
    torch.cuda.synchronize()
    rz, ru = O.flow_noise(z0[:, :n], eps[:, :n], t)
    _check(_f64(zt[:, :n]), rz, c["dtype"], "z_t")
    _check(_f64(u[:, :n]), ru, c["dtype"], "target")
    # t = 0 and t = 1 give the noise and the clean latent exactly
    assert np.array_equal(_f64(zt[0, :n]), eps[0, :n])
    assert np.array_equal(_f64(zt[-1, :n]), z0[-1, :n])
    # the padding of each item is not written
    assert bool((zt[:, n:] == 3.0).all()) and bool((u[:, n:] == 3.0).all())


@pytest.mark.parametrize("case", list(CASES))
def test_flow_loss(M, case):
    c = CASES[case]
    (z0, eps, v), (dz0, deps, dv), _ = _tensors(c, 12)
    n = c["n"]
    loss = torch.empty(c["batch"], dtype=torch.float32, device="cuda")
    nw = M.flow_loss_workspace_size(c["batch"], n)
    ws = torch.empty(nw, dtype=torch.uint8, device="cuda")
    M.flow_loss(dv[:, :n], dz0[:, :n], deps[:, :n], loss, ws, nw)
    torch.cuda.synchronize()
    ref = O.flow_loss(v[:, :n], z0[:, :n], eps[:, :n])
    got = loss.cpu().numpy().astype(np.float64)
    assert np.allclose(got, ref, rtol=1e-5, atol=0), (got, ref)
    # the summation order is fixed: a second call gives the same bits
    loss2 = torch.empty_like(loss)
    M.flow_loss(dv[:, :n], dz0[:, :n], deps[:, :n], loss2, ws, nw)
    torch.cuda.synchronize()
    assert torch.equal(loss, loss2)


def test_flow_single_output_and_errors(M):
    c = CASES["ragged_bf16"]
    (z0, eps, _), (dz0, deps, _), t = _tensors(c, 13)
    n = c["n"]
    td = torch.from_numpy(t).cuda()
    u = torch.full_like(dz0, 3.0)
    M.flow_noise(dz0[:, :n], deps[:, :n], td, None, u[:, :n])  # target only
    torch.cuda.synchronize()
    _check(_f64(u[:, :n]), z0[:, :n] - eps[:, :n], "bf16", "target only")
    with pytest.raises(M.MmditError):  # nothing to write
        M.flow_noise(dz0[:, :n], deps[:, :n], td, None, None)
    loss = torch.empty(c["batch"], dtype=torch.float32, device="cuda")
    with pytest.raises(M.MmditError):  # no workspace
        M.flow_loss(dz0[:, :n], dz0[:, :n], deps[:, :n], loss)
