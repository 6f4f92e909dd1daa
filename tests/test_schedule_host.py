"""Host checks of the attention kernels' work schedules (no GPU).

The forward launches either one CTA per fold (query-tile pairs n_pairs-1-f and f of one group)
or, when that grid's last wave would be mostly empty and K and V fit in L2, a persistent grid
that walks all pairs heaviest first in a snake order.  The backward launches one CTA per fold
(key tiles f and n_kt-1-f) or, for short folds, a persistent grid that takes folds by stride.
These tests restate the launch choice and the per-CTA item sequence of
csrc/s2attn_fwd_sm100.cu and csrc/s2attn_bwd_sm100.cu and check, for many shapes and SM
counts, that every work item is visited exactly once; the GPU parity tests check the kernels.
"""
import collections

import pytest


def fwd_schedule(B, N, H, G, n_sm, D=128):
    """(snake, grid, items per CTA as lists of (unit, pair))."""
    n_qt = G // 128
    n_pairs = (n_qt + 1) // 2
    n_units = B * H * (N // G)
    n_fold = (n_pairs + 1) // 2
    folds = n_fold * n_units
    waves = (folds + n_sm - 1) // n_sm
    kv_bytes = 2.0 * B * N * H * D * 2
    snake = folds * 10 < waves * n_sm * 9 and kv_bytes <= 160e6
    n_items = n_pairs * n_units
    grid = min(n_items, n_sm) if snake else folds
    per_cta = []
    for cta in range(grid):
        items = []
        r = 0
        while True:
            if snake:
                i = r * grid + ((grid - 1 - cta) if r & 1 else cta)
                if i >= n_items:
                    break
                unit, m = i % n_units, n_pairs - 1 - i // n_units
            else:
                fi, unit = cta % n_fold, cta // n_fold
                if r > 1 or (r == 1 and fi == n_pairs - 1 - fi):
                    break
                m = n_pairs - 1 - fi if r == 0 else fi
            items.append((unit, m))
            r += 1
        per_cta.append(items)
    return snake, grid, per_cta


def bwd_schedule(B, N, H, G, n_sm):
    """(persistent, grid, items per CTA as lists of (unit, key tile))."""
    n_kt = G // 128
    n_fold = (n_kt + 1) // 2
    folds = n_fold * B * H * (N // G)
    persistent = n_kt % 2 == 0 and n_kt <= 32
    grid = min(folds, n_sm) if persistent else folds
    per_cta = []
    for cta in range(grid):
        items = []
        it = 0
        while True:
            if persistent:
                f, sub = cta + (it >> 1) * grid, it & 1
                if f >= folds:
                    break
            else:
                f, sub = cta, it
                if sub > 1:
                    break
            fi, unit = f % n_fold, f // n_fold
            if sub == 1 and fi == n_kt - 1 - fi:
                break
            items.append((unit, n_kt - 1 - fi if sub else fi))
            it += 1
        per_cta.append(items)
    return persistent, grid, per_cta


SHAPES = [
    # (B, N, H, G)
    (1, 8192, 32, 2048),      # 7B@8k: forward snake, backward persistent
    (1, 32768, 32, 8192),     # 7B@32k: folded grids
    (1, 32768, 32, 4096),
    (1, 16384, 32, 2048),
    (2, 768, 2, 256),
    (1, 768, 2, 384),         # odd number of query / key tiles per group
    (1, 384, 1, 384),         # one group of three tiles
    (1, 8192, 8, 512),
    (1, 8192, 18, 512),
    (3, 4096, 5, 1024),
    (1, 102400, 32, 25600),
    (1, 65536, 40, 16384),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("n_sm", [1, 7, 148, 1000])
def test_forward_visits_every_pair_once(shape, n_sm):
    B, N, H, G = shape
    _, grid, per_cta = fwd_schedule(B, N, H, G, n_sm)
    n_pairs = (G // 128 + 1) // 2
    n_units = B * H * (N // G)
    seen = collections.Counter(item for items in per_cta for item in items)
    assert set(seen) == {(u, m) for u in range(n_units) for m in range(n_pairs)}
    assert max(seen.values()) == 1
    assert grid >= 1


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("n_sm", [1, 7, 148, 1000])
def test_backward_visits_every_key_tile_once(shape, n_sm):
    B, N, H, G = shape
    _, grid, per_cta = bwd_schedule(B, N, H, G, n_sm)
    n_kt = G // 128
    n_units = B * H * (N // G)
    seen = collections.Counter(item for items in per_cta for item in items)
    assert set(seen) == {(u, kt) for u in range(n_units) for kt in range(n_kt)}
    assert max(seen.values()) == 1
    assert grid >= 1


def test_schedule_choices_on_the_workloads():
    # the 8k workload takes the forward snake and the backward's persistent grid; 32k and larger
    # take one CTA per fold in both kernels
    assert fwd_schedule(1, 8192, 32, 2048, 148)[0] is True
    assert bwd_schedule(1, 8192, 32, 2048, 148)[0] is True
    for shape in ((1, 32768, 32, 8192), (1, 65536, 40, 16384), (1, 102400, 32, 25600)):
        assert fwd_schedule(*shape, 148)[0] is False
        assert bwd_schedule(*shape, 148)[0] is False


def test_forward_snake_balances_the_8k_workload():
    # work of pair m: 2m+2 K/V steps plus about one step of per-item overhead; the folded grid
    # (512 equal CTAs on 148 SMs, 3.46 waves) reaches 0.865 of perfect balance, the snake > 0.95
    snake, grid, per_cta = fwd_schedule(1, 8192, 32, 2048, 148)
    assert snake and grid == 148
    loads = [sum(2 * m + 2 + 1 for _, m in items) for items in per_cta]
    assert sum(loads) / len(loads) / max(loads) > 0.95
