"""The seeded generator: host C twin == torch path, counters are position-stable,
and the draws have the stated moments."""

import numpy as np
import torch

import synth


def test_c_and_torch_paths_give_identical_bits():
    for dt in (torch.float32, torch.bfloat16):
        for off in (0, 12345, (1 << 32) - 3):
            a = synth.normal((37, 129), 7, 11, 0.02, dt, offset=off)
            b = synth.normal((37, 129), 7, 11, 0.02, dt, offset=off, use_c=False)
            assert torch.equal(a.view(torch.int16 if dt == torch.bfloat16 else torch.int32),
                               b.view(torch.int16 if dt == torch.bfloat16 else torch.int32))


def test_token_rows_do_not_depend_on_batch():
    big = synth.tokens(40, 256, seed=3)
    assert torch.equal(synth.tokens(7, 256, seed=3, first_token=20), big[20:27])


def test_moments_and_zipf_prior():
    x = synth.normal((1 << 20,), 0, 99, 1.0, torch.float32).double()
    assert abs(x.mean().item()) < 5e-3 and abs(x.std().item() - 1.0) < 5e-3
    b = synth.zipf_logit_bias(384, 1.1, seed=0).double()
    assert abs(torch.exp(b).sum().item() - 1.0) < 1e-6
    rank = synth.zipf_permutation(384, 0)
    assert sorted(rank.tolist()) == list(range(1, 385))
    p = np.exp(b.numpy())
    assert np.argmax(p) == int(np.where(rank == 1)[0][0])
