"""Pins of the parameter contract against the pages
(tests/golden/lcsa_parameters.txt: the printed topk_ratio formula evaluated at
four sizes, and the printed latent geometry), and of the block budget reading."""
import os

import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lcsa_parameters.txt")


def golden(kind):
    with open(GOLDEN) as f:
        for line in f:
            parts = line.split()
            if parts and parts[0] == kind:
                yield [float(p) for p in parts[1:]]


@pytest.mark.parametrize("H,W,sr,ratio", list(golden("topk")))
def test_topk_ratio_rule(H, W, sr, ratio):
    # k = floor(topk_ratio * blocks per latent frame); token grid = pixels / 16
    gh, gw = int(H) // 16, int(W) // 16
    for bh, bw in ((8, 16), (8, 8)):
        if gw % bw:
            continue
        bpf = (gh // bh) * (gw // bw)
        k = oracle.resolve_topk(sr, gh, gw, 1, bh, bw)
        assert k == int(ratio * bpf + 1e-9)
        # the budget is independent of the resolution in blocks x tokens
        assert k == int(sr * 3840 / (bh * bw) + 1e-9)


@pytest.mark.parametrize("H,W,frames,lh,lw,tokens", list(golden("grid")))
def test_latent_grid(H, W, frames, lh, lw, tokens):
    assert (H / 8, W / 8) == (lh, lw)                # 8x VAE
    assert frames * (lh / 2) * (lw / 2) == tokens    # 2x2 patchify


def test_budget_of_the_measured_workloads():
    from block_sparse_video_lcsa_b200 import synth
    want = {"stream_768x1280": 60, "first_768x1280_sr2": 60, "first_768x1280_sr1.5": 45,
            "stream_768x1408": 120, "stream_2176x3840": 60}
    for name, k in want.items():
        g = oracle.Geometry.from_workload(synth.WORKLOADS[name])
        assert g.topk == k, name


def test_budget_is_floored():
    """The budget reading takes the floor of topk_ratio * blocks per latent
    frame: at 768x1280 (30 blocks of 128 tokens per frame) sparse_ratio 1.55
    gives 46.5 blocks -> 46; at 768x1408 (66 blocks of 64 tokens) sparse_ratio
    1.01 gives 60.6 -> 60."""
    assert oracle.resolve_topk(1.55, 48, 80, 1, 8, 16) == 46
    assert oracle.resolve_topk(1.01, 48, 88, 1, 8, 8) == 60
