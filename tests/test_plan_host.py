"""Launch planning of the real scan on the host (no GPU): over a sweep of shapes, the backward's
workspace stays within its caps and the launch counts have the structure the planner promises."""
import itertools
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists(
    os.path.join(ROOT, "selective_state_space_bwd_b200", "libssm_scan.so")),
    reason="needs nvcc or a prebuilt libssm_scan.so")


@pytest.fixture(scope="module")
def S():
    from selective_state_space_bwd_b200 import build, ssm_scan
    build.build()
    ssm_scan.lib()
    return ssm_scan


def _shapes():
    for B, L, D in itertools.product((1, 2, 4, 8, 16), (1, 127, 2048, 8192), (32, 1024, 1536, 4096)):
        yield B, L, D
    yield 1, 128000, 1024
    yield 1, 512000, 1024


@pytest.mark.parametrize("B,L,D", list(_shapes()))
def test_backward_plan_caps_and_launches(S, B, L, D):
    N, T = 16, 128
    shp = S.real_shape(B, L, D, N, T, S.SSM_BF16)
    ckpt = S.checkpoint_bytes(shp)
    cap = max(ckpt, 128 << 20)
    bw = S.workspace_bytes(shp, True)
    # capped dB/dC partial sums + scratch slots (592 x 96 KB at most) + segment summaries (at
    # most the checkpoints) + small per-(batch, segment) sums
    assert bw <= 2 * cap + (193 << 20)
    nf, nb = S.kernel_launches(shp, False), S.kernel_launches(shp, True)
    # forward: one scan launch, or summary + carry + scan when split in time
    assert nf in (1, 3)
    # backward: [summary + carry] + k x (main + dB/dC reduction) + parameter reduction
    assert nb >= 3 and nb % 2 == 1
    # a grid that already fills the SMs (>= 296 CTAs of 32 channels) never splits the forward
    if B * (-(-D // 32)) >= 296:
        assert nf == 1


def test_backward_workspace_grows_no_faster_than_checkpoints(S):
    """The backward's partial-sum buffer is capped at max(checkpoint bytes, 128 MiB) per launch:
    a wide problem's workspace grows with L no faster than its checkpoints (O(L/T)), and the
    sequence is walked in more launches once the 128 MiB floor binds."""
    a = S.real_shape(16, 8192, 4096, 16, 128, S.SSM_BF16)
    b = S.real_shape(16, 32768, 4096, 16, 128, S.SSM_BF16)
    assert S.workspace_bytes(b, True) - S.workspace_bytes(a, True) <= S.checkpoint_bytes(b) - S.checkpoint_bytes(a)
    c = S.real_shape(4, 2048, 4096, 16, 128, S.SSM_BF16)   # partials of the whole sequence fit
    d = S.real_shape(4, 16384, 4096, 16, 128, S.SSM_BF16)  # 128 MiB floor binds: more launches
    assert S.kernel_launches(d, True) > S.kernel_launches(c, True)
    assert S.workspace_bytes(d, True) <= (128 << 20) + (193 << 20) + S.checkpoint_bytes(d)
