"""GPU parity of the per-denoising-step path (``StepPipeline``): host list build into a pinned ring buffer,
asynchronous upload on the stream, kernel launch -- fifty steps queued without a host synchronisation, each
step's output kept and compared with the fp64 oracle given that step's lists.

The anchors move one frame per step (techwalker article "华为巴黎研究院让AI视频“不再原地打转”", section 三), so a
race in the pipeline (a list buffer rewritten before its copy, a copy landing while a kernel still reads the
device buffer, the wrong stream) would give a step the lists of another step; the negative control shows that
another step's lists are told apart.
"""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import lists as OL

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def test_fifty_pipelined_steps_against_oracle(gpu_lib):
    import synthetic
    from block_sparse_attention_frame_b200.pipeline import StepPipeline

    T, C, W, P, H, d = 121, 21, 9, 64, 2, 128
    q, k, v = synthetic.make_custom(T, P, H, d, seed=121, device="cuda")
    pipe = StepPipeline(T, C, W, P, "cuda")
    outs = []
    for s in range(50):
        outs.append(pipe.step(s, q, k, v, torch.empty_like(q)))
    torch.cuda.synchronize()
    assert gpu_lib.lvsa_get_device_status(clear=True) == 0
    assert len(pipe.build_us) == 50
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    g = np.random.default_rng(7)
    frames = sorted(set([0, 1, 60, 119, 120] + [int(f) for f in g.choice(T, 4, replace=False)]))
    rows = [f * P + r for f in frames for r in range(P)]
    for s in range(50):
        got = outs[s][:, rows].float().cpu().numpy()
        ref = OA.sparse_attention_rows(qc, kc, vc, OL.frame_lists(T, C, W, s), P, rows)
        err = np.abs(got - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (s, err.max(), err.mean())
        # negative control: the lists of the next step (anchors one frame further) miss by far
        wrong = OA.sparse_attention_rows(qc, kc, vc, OL.frame_lists(T, C, W, s + 1), P, rows)
        assert np.abs(got - wrong).mean() > 5 * MEAN_ABS, s


def test_fixed_grid_pipeline_repeats_step_zero(gpu_lib):
    """Fixed-grid ablation: every step attends the step-0 pattern, so every step's output is the same bits."""
    import synthetic
    from block_sparse_attention_frame_b200.pipeline import StepPipeline

    T, C, W, P, H, d = 30, 7, 3, 130, 2, 64
    q, k, v = synthetic.make_custom(T, P, H, d, seed=30, device="cuda")
    pipe = StepPipeline(T, C, W, P, "cuda", fixed_grid=True, depth=3)
    outs = [pipe.step(s, q, k, v, torch.empty_like(q)) for s in range(8)]
    rp = StepPipeline(T, C, W, P, "cuda")  # kept alive until its copies are done
    rot = rp.step(5, q, k, v, torch.empty_like(q))
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    assert not torch.equal(rot.view(torch.int16), outs[0].view(torch.int16))
    ref = OA.sparse_attention(q.cpu(), k.cpu(), v.cpu(), OL.frame_lists(T, C, W, 0), P)
    err = np.abs(outs[5].float().cpu().numpy() - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


def test_pipeline_on_a_side_stream(gpu_lib):
    """Steps queued on a non-default stream, the outputs read after that stream's work: same bits as the
    plain call with each step's lists."""
    import synthetic
    from block_sparse_attention_frame_b200.pipeline import StepPipeline

    T, C, W, P, H, d = 12, 5, 2, 300, 3, 128
    q, k, v = synthetic.make_custom(T, P, H, d, seed=12, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    pipe = StepPipeline(T, C, W, P, "cuda", depth=2)
    outs = [pipe.step(s, q, k, v, torch.empty_like(q), stream=side) for s in range(6)]
    torch.cuda.current_stream().wait_stream(side)
    for s, o in enumerate(outs):
        lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, C, W, s)).cuda()
        ref = gpu_lib.lvsa_attention(q, k, v, lists, P)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), s
