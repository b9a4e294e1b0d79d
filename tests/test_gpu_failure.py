"""Failure detection on the GPU without faulting it: a bounded device wait
runs out on an mbarrier that nothing arrives at (a 50 ms limit); the kernel
records MMDIT_ETIMEOUT and returns; the host reads the status, the flag
clears, kernels launched while it was set skip their work, and the context
stays usable for a correct attention call afterwards."""
import math

import numpy as np
import pytest

import oracle as O
from joint_video_audio_rope_b200 import workloads as WL

from _util import assert_close, to_device, to_host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from joint_video_audio_rope_b200 import build
    build.build()
    from joint_video_audio_rope_b200 import mmdit
    return mmdit


def _small():
    w = WL.Workload("fail", [WL.video(3, 6, 10), WL.text(20)], batch=1, heads=2, head_dim=128,
                    dtype="bf16", seed=77, qk_std=WL.INV_SQRT_128, v_std=WL.INV_SQRT_128)
    x = WL.generate(w)
    return w, x, {n: to_device(x[n], "bf16") for n in ("q", "k", "v")}


@pytest.fixture()
def clear_flag(M):
    yield
    M.device_status()  # whatever happened, leave the device error word clear


def test_bounded_wait_times_out_and_context_survives(M, clear_flag):
    assert M.device_status() == M.OK
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.selftest_wait_timeout(50, waited)
    torch.cuda.synchronize()
    assert int(waited.item()) == 1
    # while the flag is set, attention kernels skip their work
    w, x, dev = _small()
    o = torch.full_like(dev["q"], 7.0)
    M.joint_attn(dev["q"], dev["k"], dev["v"], o, M.desc_of(dev["q"]), M.make_layout(w.segments),
                 1 / math.sqrt(128))
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)
    assert M.device_status() == M.ETIMEOUT
    assert "bounded device wait" in M.last_error()
    assert M.device_status() == M.OK  # read-and-clear
    # the context is usable: the same call now computes the right answer
    M.joint_attn(dev["q"], dev["k"], dev["v"], o, M.desc_of(dev["q"]), M.make_layout(w.segments),
                 1 / math.sqrt(128))
    torch.cuda.synchronize()
    assert M.device_status() == M.OK
    host = {n: WL.as_f64(x[n], "bf16") for n in ("q", "k", "v")}
    ref, _ = O.joint_attn(host["q"], host["k"], host["v"], 1 / math.sqrt(128))
    assert_close(to_host_f64(o), ref, "bf16", "after timeout")


def test_selftest_rejects_bad_limits(M):
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, 5000):
        with pytest.raises(M.MmditError) as e:
            M.selftest_wait_timeout(bad, waited)
        assert e.value.status == M.EINVAL
