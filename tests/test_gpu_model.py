"""The whole-model driver (statistics of every linear, trace-sensitivity bit
allocation, then BiIP + solver + loss per linear) on one 7B-shaped block with
few tokens, checked against the oracle where the oracle can follow it: the
allocation of bits from the same scores, and scores that separate q/k/v
(same inputs, different gradients)."""
import math

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu


def test_one_block_model():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA GPU")
    from post_weight_quantization_syrk_b200.model import SHAPE, synthetic_model
    r = synthetic_model(n_tokens=2048, n_blocks=1).run()
    pl = r["per_linear"]
    assert len(pl) == 7 and r["weights"] == sum(SHAPE[x["linear"]][0] * SHAPE[x["linear"]][1] for x in pl)
    scores = [x["score"] for x in pl]
    n = [SHAPE[x["linear"]][0] * SHAPE[x["linear"]][1] for x in pl]
    assert [x["bits"] for x in pl] == list(O.allocate_bits(scores, n, (2, 3, 4), 3.0))
    assert r["average_bits"] <= 3.0 + 1e-12
    # q, k, v share H_X but not H_G: the joint score tells them apart
    trX = {x["linear"]: x["tr_X"] for x in pl}
    assert trX["q"] == trX["k"] == trX["v"]
    assert len({x["score"] for x in pl if x["linear"] in "qkv"}) == 3
    for x in pl:
        assert math.isfinite(x["loss"]) and x["loss"] > 0
        assert abs(x["score"] - x["tr_X"] * x["tr_G"]) <= 1e-12 * abs(x["score"])
    assert r["gpu_seconds"] > 0


def test_overlapped_linears_match_sequential():
    """Pass 2 runs each linear on a second stream once its input group's
    factor is ready; two blocks (buffers freed and reused across the join)
    must give exactly the bits and losses of the one-stream order."""
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA GPU")
    from post_weight_quantization_syrk_b200.model import synthetic_model
    a = synthetic_model(n_tokens=2048, n_blocks=2, overlap=True).run()
    b = synthetic_model(n_tokens=2048, n_blocks=2, overlap=False).run()
    assert len(a["per_linear"]) == len(b["per_linear"]) == 14
    for x, y in zip(a["per_linear"], b["per_linear"]):
        assert (x["block"], x["linear"], x["bits"]) == (y["block"], y["linear"], y["bits"])
        assert x["loss"] == y["loss"], (x, y)
    assert a["gpu_seconds"] > 0 and b["gpu_seconds"] > 0
