"""Parser for the hand-computed plan fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _matrix(lines, P, dtype):
    return np.array([[int(x) for x in lines.pop(0).split()] for _ in range(P)], dtype=dtype)


def load_plan_fixture(name="plan_4x4.txt", with_group=False):
    """Returns (P, [dict(step, plan, expect, hit, age)]), or (P, g, cases)
    with ``with_group`` (a fixture without a "g" line has g = 1)."""
    with open(os.path.join(GOLDEN, name)) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]
    assert lines[0].startswith("P ")
    P = int(lines.pop(0).split()[1])
    g = 1
    if lines[0].startswith("g "):
        g = int(lines.pop(0).split()[1])
    cases = []
    while lines:
        head = lines.pop(0)
        assert head.startswith("step "), head
        case = {"step": int(head.split()[1])}
        assert lines.pop(0) == "plan"
        case["plan"] = _matrix(lines, P, np.uint8)
        case["expect"] = lines.pop(0).split()[1]
        if case["expect"] == "ok":
            assert lines.pop(0) == "hit"
            case["hit"] = _matrix(lines, P, np.uint8)
            assert lines.pop(0) == "age"
            case["age"] = _matrix(lines, P, np.int32)
        cases.append(case)
    if with_group:
        return P, g, cases
    return P, cases


def load_select_fixture(name="select_4x4.txt"):
    """Returns (P, window, ase [P,P] float64, [(ratio, plan [P,P] uint8)])."""
    with open(os.path.join(GOLDEN, name)) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]
    P = int(lines.pop(0).split()[1])
    window = int(lines.pop(0).split()[1])
    assert lines.pop(0) == "ase"
    ase = np.array([[float(x) for x in lines.pop(0).split()] for _ in range(P)])
    cases = []
    while lines:
        ratio = float(lines.pop(0).split()[1])
        cases.append((ratio, _matrix(lines, P, np.uint8)))
    return P, window, ase, cases
