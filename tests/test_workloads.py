"""The seeded input generators shared by the CUDA path and the oracle: they
hold no method arithmetic, but both sides depend on their shapes, seeds and
distributions."""
import itertools

import numpy as np
import torch

from video_diffusion_transformer_rms_b200.workloads import (WORKLOADS, _TENSOR_IDS, activation,
                                                            make_inputs, outlier_columns,
                                                            seed_for, to_oracle_array,
                                                            vectors)


def test_shapes_of_the_named_workloads():
    rows = {n: w.rows for n, w in WORKLOADS.items()}
    assert rows == {"tiny": 56, "medium": 8264, "clip5s": 126552, "clip15s": 371592,
                    "cfg5s": 2 * 126552, "cfg5s_d3072": 2 * 126552}
    c = WORKLOADS["clip5s"]
    assert (c.T, c.H, c.W, c.n_audio, c.D) == (31, 48, 84, 1560, 5120)
    assert c.n_video == 124992 and c.bytes_per_row() == {
        "rms_adaln": 20480, "gate_residual": 30720, "qknorm_rope3d": 40960}
    assert WORKLOADS["cfg5s_d3072"].D == 3072 and WORKLOADS["tiny"].esize == 4


def test_every_tensor_of_every_workload_has_its_own_seed():
    seeds = [seed_for(w, t) for w, t in itertools.product(WORKLOADS.values(), _TENSOR_IDS)]
    assert len(seeds) == len(set(seeds))


def test_activation_is_deterministic_with_seeded_outlier_columns():
    a = activation(300, 5120, torch.float32, "cpu", 7, outliers=True)
    b = activation(300, 5120, torch.float32, "cpu", 7, outliers=True)
    c = activation(300, 5120, torch.float32, "cpu", 8, outliers=True)
    assert torch.equal(a, b) and not torch.equal(a, c)
    cols = outlier_columns(5120, 7)
    assert cols.numel() == 51 and torch.equal(cols, torch.sort(torch.unique(cols)).values)
    std = a.std(dim=0)
    mask = torch.zeros(5120, dtype=torch.bool)
    mask[cols] = True
    assert 15.0 < float(std[mask].mean()) < 25.0      # scaled by 20
    assert 0.9 < float(std[~mask].mean()) < 1.1       # N(0, 1)
    plain = activation(300, 5120, torch.float32, "cpu", 7, outliers=False)
    assert 0.95 < float(plain.std()) < 1.05


def test_vectors_mean_and_std():
    v = vectors((200_000,), 1.0, 0.1, torch.float32, "cpu", 3)
    assert abs(float(v.mean()) - 1.0) < 2e-3 and abs(float(v.std()) - 0.1) < 2e-3


def test_inputs_are_rounded_once_to_the_io_dtype_and_copied_exactly():
    t = make_inputs(WORKLOADS["tiny"], "cpu")
    assert t["x"].dtype == torch.float32 and t["qkv"].shape == (56, 3 * 256)
    x = activation(4, 16, torch.bfloat16, "cpu", 11, outliers=False)
    bits = to_oracle_array(x)
    assert bits.dtype == np.uint16
    back = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    assert torch.equal(back, x)
