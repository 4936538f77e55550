"""GPU parity of the joint video + text call (lvsa_attention_joint) against the fp64 oracle
(oracle.attention.joint_attention).  Reading of the pages (silent on non-video tokens): video rows attend
their frames' lists plus every text token, text rows attend every token.  Same tolerance as the video-only
call: max-abs <= 2e-2 and mean-abs <= 2e-3 on small cases; on a full-size call, sampled rows with the
relative mean bound and a negative control."""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import lists as OL

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_MEAN = 1e-2


def test_no_text_tokens_is_the_video_call_bit_for_bit(gpu_lib):
    import synthetic

    q, k, v = synthetic.make_custom(6, 300, 3, 128, seed=2, device="cuda")
    lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(6, 4, 2, 1)).cuda()
    a = gpu_lib.lvsa_attention(q, k, v, lists, 300)
    b = gpu_lib.lvsa_attention_joint(q, k, v, lists, 300)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


JOINT_CASES = [
    (8, 64, 32, 2, 64, 4, 2, 3),      # the tiny shape with a short prompt
    (6, 300, 77, 3, 128, 4, 2, 1),    # straddling video blocks, one partial text tile
    (5, 256, 300, 2, 128, 3, 2, 2),   # two text blocks (256 + 44 rows), three text tiles
    (4, 100, 130, 2, 64, 3, 1, 0),    # frames shorter than a block (blocks stay inside a frame)
    (9, 200, 1, 2, 128, 5, 2, 4),     # a single text token
    (3, 1560, 256, 1, 128, 2, 1, 0),  # video-sized frames
    (1, 500, 60, 2, 128, 1, 1, 0),    # T = 1: one frame and a prompt
]


# every case at batch 1, the smaller ones also at batch 2
@pytest.mark.parametrize("T,P,n_text,H,d,C,W,step,B",
                         [c + (1,) for c in JOINT_CASES] + [c + (2,) for c in JOINT_CASES if c[0] * c[1] <= 2000])
def test_joint_matches_oracle(gpu_lib, T, P, n_text, H, d, C, W, step, B):
    import synthetic

    q, k, v = synthetic.make_joint(T, P, n_text, H, d, B=B, seed=T + n_text, device="cpu")
    lists_np = gpu_lib.lvsa_build_frame_lists(T, C, W, step)
    out = gpu_lib.lvsa_attention_joint(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(lists_np).cuda(), P)
    torch.cuda.synchronize()
    assert gpu_lib.lvsa_get_device_status(clear=True) == 0
    got = out.float().cpu().numpy()
    ref = OA.joint_attention(q, k, v, OL.frame_lists(T, C, W, step), P, T)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    if n_text >= 32:
        # negative control: the video-only oracle on the video rows must differ (the text tokens count; one
        # text token among ~1000 keys moves the outputs by less than the tolerance, so that case is skipped)
        ref_video = OA.sparse_attention(q[:, :T * P], k[:, :T * P], v[:, :T * P], OL.frame_lists(T, C, W, step), P)
        assert np.abs(got[:, :T * P] - ref_video).mean() > MEAN_ABS


def test_full_size_joint_call_sampled_rows(gpu_lib):
    """HunyuanVideo-1.5 1.5x shape (T = 49, P = 1560, 16 heads) with 256 text tokens: sampled video rows of
    five frames and sampled text rows against the oracle."""
    import synthetic

    T, P, n_text, H, d, C, W, step = 49, 1560, 256, 16, 128, 33, 13, 7
    q, k, v = synthetic.make_joint(T, P, n_text, H, d, seed=1005, device="cuda")
    lists_np = gpu_lib.lvsa_build_frame_lists(T, C, W, step)
    out = gpu_lib.lvsa_attention_joint(q, k, v, torch.from_numpy(lists_np).cuda(), P)
    torch.cuda.synchronize()
    assert gpu_lib.lvsa_get_device_status(clear=True) == 0
    g = np.random.default_rng(5)
    rows = []
    for t in (0, 1, T // 2, T - 2, T - 1):
        rows += [t * P, t * P + P - 1] + list(t * P + g.choice(P, 6, replace=False))
    rows += [T * P, T * P + n_text - 1] + list(T * P + g.choice(n_text, 14, replace=False))
    rows = sorted(set(int(r) for r in rows))
    lists = OL.frame_lists(T, C, W, step)
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()  # the oracle takes host tensors
    ref = OA.joint_attention_rows(qc, kc, vc, lists, P, T, rows)
    got = out[:, rows].float().cpu().numpy()
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert err.mean() <= REL_MEAN * np.abs(ref).mean(), (err.mean(), np.abs(ref).mean())
    wrong = OA.joint_attention_rows(qc, kc, vc, OL.frame_lists(T, C, W, step + 1), P, T, rows)
    video = [i for i, r in enumerate(rows) if r < T * P]
    assert np.abs(got[:, video] - wrong[:, video]).mean() > 10 * REL_MEAN * np.abs(ref).mean()
