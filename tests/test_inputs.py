"""Pins for the input generators: the Lloyd-Max grid against Max's published
16-level Gaussian quantiser, determinism, and the workload shapes."""
import numpy as np
import torch

from bit_codebook_quantized_router_b200 import inputs

# Positive output levels of the minimum-mean-square-error 16-level quantiser
# for a unit Gaussian (J. Max, "Quantizing for Minimum Distortion", IRE Trans.
# Information Theory, 1960, Table I, N = 16).
MAX_16 = np.array([0.1284, 0.3881, 0.6568, 0.9424, 1.2562, 1.6181, 2.0690, 2.7326])


def test_lloyd_grid_matches_max_table_within_sampling_error():
    g = inputs.lloyd_max_grid(0)
    assert g.dtype == np.float32 and np.all(np.diff(g) > 0)
    assert np.max(np.abs(g - MAX_16)) < 0.03


def test_lloyd_iteration_converges_to_max_table_on_a_large_sample():
    g = inputs.lloyd_max_grid(1, n_samples=2_000_000, tol=1e-10)
    assert np.max(np.abs(g - MAX_16)) < 0.01


def test_generators_are_deterministic_and_shaped():
    w = inputs.WORKLOADS["tiny"]
    a = inputs.expert_weight(w, 3, "down")
    b = inputs.expert_weight(w, 3, "down")
    assert a.dtype == torch.bfloat16 and a.shape == (w.shape.H, w.shape.I)
    assert torch.equal(a, b)
    assert not torch.equal(a, inputs.expert_weight(w, 4, "down"))
    assert abs(a.float().std().item() - 0.02) < 0.002
    x = inputs.activations(w)
    assert x.shape == (4, 256) and x.dtype == torch.bfloat16
    lg = inputs.router_logits(w)
    assert lg.shape == (4, 8) and lg.dtype == torch.float32


def test_mixed_tables_flag_the_defect_experts():
    tables, tid = inputs.layer_tables(inputs.WORKLOADS["prefill_t8192"])
    assert tables.shape == (2, 8)
    assert np.array_equal(tables[1], inputs.E2M1_TABLE)
    assert sorted(np.nonzero(tid)[0].tolist()) == [15, 30, 86, 139, 164]
