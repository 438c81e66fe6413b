"""The oracle against the hand-derived worked examples in tests/golden/."""
import json
import math
import os

import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURES = json.load(open(os.path.join(HERE, "golden", "closed_forms.json")))

_NAMES = {"ln2": math.log(2.0), "ln3": math.log(3.0)}


def _num(s):
    if isinstance(s, (int, float)):
        return float(s)
    for fn in ("cos", "sin"):
        if fn in s:
            sign = -1.0 if s.startswith("-") else 1.0
            arg = float(s[s.index("(") + 1:s.index(")")])
            return sign * getattr(math, fn)(arg)
    return _NAMES[s] if s in _NAMES else float(s)


@pytest.mark.parametrize("case", FIXTURES["decode"], ids=lambda c: c["name"])
def test_decode_closed_form(case):
    q = torch.tensor(case["q"], dtype=torch.float32)            # [Hq, d]
    K = torch.tensor(case["K"], dtype=torch.float32)            # [L, Hkv, d]
    V = torch.tensor(case["V"], dtype=torch.float32)
    L, Hkv, d = K.shape
    kp = torch.zeros(1, Hkv, 16, d)
    vp = torch.zeros(1, Hkv, 16, d)
    kp[0, :, :L] = K.permute(1, 0, 2)
    vp[0, :, :L] = V.permute(1, 0, 2)
    out = oracle.paged_attention_decode(q[None], kp, vp, torch.zeros(1, 1, dtype=torch.int32),
                                        torch.tensor([L], dtype=torch.int32), _num(case["scale"]))
    want = torch.tensor([[_num(x) for x in row] for row in case["expected"]], dtype=torch.float64)
    assert (out[0] - want).abs().max().item() < 1e-13


@pytest.mark.parametrize("case", FIXTURES["rope"], ids=lambda c: c["name"])
def test_rope_closed_form(case):
    x = torch.tensor([case["x"]], dtype=torch.float64)
    got = oracle.rope(x, torch.tensor([case["pos"]]), case["theta"])[0]
    want = torch.tensor([_num(v) for v in case["expected"]], dtype=torch.float64)
    assert (got - want).abs().max().item() < 1e-13
