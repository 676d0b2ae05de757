"""The backward's checkpoint-slot arithmetic, restated on the CPU: sequence n
(tokens start_n .. start_n + len_n) owns slots start_n // 64 + n + c for its
chunks c < ceil(len_n / 64). The kernels index the fp32 checkpoint arrays with
it and the workspace holds tokens // 64 + N slots; these checks are the
in-bounds argument, for valid offsets and for the clamped malformed ones."""
import numpy as np
import pytest

C = 64


def clamp_bounds(cu, tokens):
    """The kernels' reading of packed offsets: each clamped to [0, tokens]."""
    out = []
    for n in range(len(cu) - 1):
        s = min(max(int(cu[n]), 0), tokens)
        e = min(max(int(cu[n + 1]), s), tokens)
        out.append((s, e - s))
    return out


def slots_used(bounds):
    used = []
    for n, (s, ln) in enumerate(bounds):
        base = s // C + n
        used.append(set(range(base, base + -(-ln // C))))
    return used


@pytest.mark.parametrize("seed", range(20))
def test_slots_of_valid_packed_batches_are_disjoint_and_in_range(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 200))
    lengths = rng.integers(0, 700, size=N) * (rng.random(N) > 0.1)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    tokens = int(cu[-1])
    used = slots_used(clamp_bounds(cu, tokens))
    limit = tokens // C + N
    seen = set()
    for s in used:
        assert not (s & seen)
        assert all(0 <= x < limit for x in s)
        seen |= s


@pytest.mark.parametrize("B,T", [(1, 1), (4, 2048), (3, 63), (2, 65), (5, 0), (7, 130)])
def test_slots_of_fixed_length_batches(B, T):
    bounds = [(n * T, T) for n in range(B)]
    used = slots_used(bounds)
    limit = (B * T) // C + B
    seen = set()
    for s in used:
        assert not (s & seen) and all(0 <= x < limit for x in s)
        seen |= s


@pytest.mark.parametrize("seed", range(10))
def test_slots_stay_in_range_for_malformed_offsets(seed):
    """Non-monotone or out-of-range offsets may make sequences share slots
    (wrong results, by contract), but never index outside the array."""
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(1, 50))
    tokens = int(rng.integers(0, 5000))
    cu = rng.integers(-100, tokens + 200, size=N + 1)
    limit = tokens // C + N
    for s in slots_used(clamp_bounds(cu, tokens)):
        assert all(0 <= x < limit for x in s)
