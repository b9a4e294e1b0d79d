"""The device-checked debug build (build --device-checks): indices read from
caller data are checked on the device, and an out-of-range one is recorded as
MMDIT_EDEVCHECK in the device error word and skipped -- nothing traps, and the
context stays usable (while the word is set, later attention kernels skip
their work, as after a timed-out wait; mmdit_device_status reads and clears
it).  The regular build skips the same index silently.

Each case runs in a child process that loads one build of the library (the
binding loads its library once per process).  The bad input is a block list
with an id past the number of blocks: the union kernel reads it, checks it,
and never uses it as an address."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import math, sys
    import numpy as np, torch
    sys.path.insert(0, {root!r})
    from joint_video_audio_rope_b200 import mmdit as M, workloads as WL
    w = WL.Workload("dc", [WL.video(4, 8, 8, order=WL.ORDER_BLOCK444)], 1, 2, 128, "bf16", 3,
                    1.0, 1.0)
    x = WL.generate(w)
    up = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = up(x["q"]), up(x["k"]), up(x["v"])
    lay = M.make_layout(w.segments)
    d = M.desc_of(q)
    nb = M.num_blocks(lay)
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 2, nb, 1))
    cnt = np.full((1, 2, nb), nb, np.int32)
    idx[0, 1, 2, nb - 1] = nb + 5          # one id past the blocks
    n = M.sparse_attn_workspace_size(d, lay, nb)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    M.sparse_attn(q, k, v, o, d, lay, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                  nb, 1 / math.sqrt(128), ws, n)
    torch.cuda.synchronize()
    st = M.device_status()
    st2 = M.device_status()                # read and cleared: the next read is clean
    # the context is still usable: a clean call afterwards runs and reports OK
    idx[0, 1, 2, nb - 1] = nb - 1
    M.sparse_attn(q, k, v, o, d, lay, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                  nb, 1 / math.sqrt(128), ws, n)
    torch.cuda.synchronize()
    st3 = M.device_status()
    assert torch.isfinite(o.float()).all()
    print("STATUS", st, st2, st3)
""")


def _run(lib):
    env = dict(os.environ, MMDIT_LIB=lib)
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [l for l in r.stdout.splitlines() if l.startswith("STATUS")][-1]
    return tuple(int(t) for t in line.split()[1:])


def test_checked_build_reports_a_bad_block_id():
    from joint_video_audio_rope_b200 import build
    lib = build.build(device_checks=True)
    assert _run(lib) == (6, 0, 0)  # MMDIT_EDEVCHECK, then cleared, then a clean call


def test_regular_build_skips_the_same_id():
    from joint_video_audio_rope_b200 import build
    lib = build.build()
    assert _run(lib) == (0, 0, 0)
