"""The parity checks themselves (CPU only): the gradient comparison the GPU
tests use catches a single zeroed row, a tile taken from the wrong head and a
missing sequence, which a whole-tensor norm alone lets through, while passing
a gradient that differs from the oracle by 16-bit rounding."""

import numpy as np
import pytest
import torch

from attn_cases import TOL_GRAD, assert_grads, local_errors, rel_fro


def _grad(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).bfloat16().double().numpy()


def test_rounded_gradients_pass():
    w = [_grad((2, 2, 333, 64), s) for s in (1, 2, 3)]
    assert_grads([_bf16(x) for x in w], w)


def test_one_zeroed_row_is_caught_by_the_tile_check():
    w = [_grad((2, 4, 1000, 64), s) for s in (1, 2, 3)]
    g = [x.copy() for x in w]
    g[1][1, 0, 200] = 0.0
    assert rel_fro(g[1], w[1]) <= TOL_GRAD          # the whole-tensor norm misses it
    with pytest.raises(AssertionError, match="block"):
        assert_grads(g, w)


def test_tile_from_the_wrong_head_is_caught():
    w = [_grad((1, 8, 1024, 64), s) for s in (1, 2, 3)]
    g = [x.copy() for x in w]
    g[2][0, 3, 128:256] = w[2][0, 4, 128:256]
    with pytest.raises(AssertionError):
        assert_grads(g, w)


def test_packed_sequence_left_out_is_caught():
    w = [_grad((3000, 4, 80), s) for s in (1, 2, 3)]
    g = [x.copy() for x in w]
    g[0][1000:1050] = 0.0          # a 50-token sequence of every head never written
    assert rel_fro(g[0], w[0]) <= 0.15
    with pytest.raises(AssertionError):
        assert_grads(g, w)


def test_near_cancelling_blocks_use_the_floor():
    w = _grad((4, 256, 16), 7)
    w[1, :128] *= 1e-4             # a block whose true gradient nearly cancels
    g = w + 1e-3 * _grad(w.shape, 8)
    errs = dict((str(i), e) for i, e in local_errors(g, w))
    assert max(errs.values()) < TOL_GRAD
