"""The TTT-Linear scan at the edges of its sizes, against the oracle: a long sequence (4 096 full
mini-batches and a tail, one CTA carrying its state through all of them) and a grid many CTA
waves deep (2 048 chains, the last ones starting only after earlier CTAs have finished).
Tolerance as in the other bf16 parity tests: max relative L2 error 1e-2 per chain and tensor."""
import torch

import synth
from parity_util import sample_chains
from test_parity_linear import TOL_BF16, compare, compare_sampled, gpu_linear, oracle_linear

import pytest

pytestmark = pytest.mark.gpu


def test_long_sequence_4096_mini_batches_and_tail(libttt):
    w = synth.workload(1, B=1, H=2, L=16 * 4096 + 9, seed=0x10C6)
    x = synth.linear_inputs(w)
    res = gpu_linear(libttt, x, w)
    assert all(torch.isfinite(t.float()).all() for t in res)
    compare(res, oracle_linear(x, w), TOL_BF16, what="long L=65545")


def test_many_chains_several_waves(libttt):
    w = synth.workload(1, B=64, H=32, L=16 * 3 + 5, seed=0x10C7)
    x = synth.linear_inputs(w, values=False)
    res = gpu_linear(libttt, x, w)
    chains = sample_chains(w.chains, 6)
    assert w.chains - 1 in chains
    ref = oracle_linear(synth.linear_inputs(w, chains=chains), w, chains=chains)
    compare_sampled(res, ref, chains, TOL_BF16, what="2048 chains")
