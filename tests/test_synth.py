"""The seeded input generator: determinism, subsets, bf16 rounding, structure."""
import numpy as np
import torch

from block_sparse_video_sol_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        # exact ties between two bf16 values, both parities
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8,
                                  65504.0, 1e-30, -0.0, 0.0], np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = synth.bf16_bits_to_f64(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16)
                                  .double().numpy())


def test_deterministic_and_head_subsets():
    w = synth.tiny()
    a = synth.generate(w)
    b = synth.generate(w, threads=1)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    sub = synth.generate(w, heads=[1])
    for x, y in zip(a, sub):
        np.testing.assert_array_equal(x[:, :, 1:2], y)
    assert a[0].shape == (1, 1024, 2, 64) and a[0].dtype == np.uint16


def test_topic_structure_and_prefix():
    w = synth.Workload("t", B=1, H=1, N=40 + 8 * 8 * 8, D=32, grid=(8, 8, 8), n_topics=4,
                       prefix=40)
    q, k, v = (synth.bf16_bits_to_f64(x)[0, :, 0] for x in synth.generate(w))
    vid_q, vid_k = q[40:], k[40:]
    # rows of one 4x4x4 tile share a topic: their q and k means are close to 2*u
    tile = synth._tile_index(w)
    m0 = vid_q[tile == 0].mean(0)
    assert abs(np.linalg.norm(m0) - 2.0) < 0.5
    assert abs(np.linalg.norm(vid_k[tile == 0].mean(0)) - 2.0) < 0.5
    # prefix rows are plain N(0,1)
    assert abs(q[:40].mean()) < 0.1 and abs(q[:40].std() - 1) < 0.1
    assert abs(v.mean()) < 0.05 and abs(v.std() - 1) < 0.05


def test_workload_shapes():
    j = synth.h56_joint()
    assert j.N == 38247 and j.prefix == 2407 and j.N - j.prefix == 10 * 56 * 64
    assert synth.h56_sweep(32768).grid == (32, 32, 32)
    assert synth.h56_n4096().grid == (16, 16, 16)


def test_literal_workloads_of_the_gpu_tests_are_valid():
    """Every Workload(...) with literal arguments in the GPU tests builds (its grid covers
    the video rows), so a mistyped case fails here rather than on a GPU."""
    import ast
    import os
    src = open(os.path.join(os.path.dirname(__file__), "test_gpu_parity.py")).read()
    n = 0
    for node in ast.walk(ast.parse(src)):
        if isinstance(node, ast.Call) and getattr(node.func, "attr", "") == "Workload":
            try:
                args = [ast.literal_eval(a) for a in node.args]
                kw = {k.arg: ast.literal_eval(k.value) for k in node.keywords}
            except ValueError:
                continue   # arguments computed at run time
            synth.Workload(*args, **kw)
            n += 1
    assert n >= 5
