"""The GEMM kernel's work schedule, written out in Python for CPU checks.

The kernel (csrc/gemm_kernel.cuh: unit_work, work_item, tail_contributors)
deals whole output tiles round-robin to its persistent units and spreads the
k-blocks of a short last round evenly over `tail_units` units; a tile whose
k-blocks several units share is finished by the last of them to arrive.  The
functions here restate that index arithmetic from the plan tl_gemm_plan
returns, so that tests can check it on the host -- coverage of every k-block,
the contributor ranges, the partial-sum slots -- for any shape before a
kernel runs.  This is test infrastructure; it computes no GEMM arithmetic.
"""
from __future__ import annotations


def unit_items(unit: int, num_units: int, full_tiles: int, tail_tiles: int, tail_units: int, num_kb: int):
    """The (tile, kb0, kb1, tail) items unit `unit` processes, in order."""
    items = []
    t = unit
    while t < full_tiles:
        items.append((t, 0, num_kb, -1))
        t += num_units
    if unit < tail_units:
        T = tail_tiles * num_kb
        g = unit * T // tail_units
        g1 = (unit + 1) * T // tail_units
        for _ in range(2):
            if g >= g1:
                break
            r = g // num_kb
            base = r * num_kb
            end = min(g1, base + num_kb)
            items.append((full_tiles + r, g - base, end - base, r))
            g = end
        assert g == g1, "a unit's range reaches past the next tile"
    return items


def tail_contributors(r: int, tail_tiles: int, tail_units: int, num_kb: int):
    """(first, last) unit whose k-block range meets tail tile r."""
    T = tail_tiles * num_kb
    U = tail_units
    x0 = r * num_kb
    x1 = x0 + num_kb - 1
    first = ((x0 + 1) * U + T - 1) // T - 1
    last = ((x1 + 1) * U + T - 1) // T - 1
    return first, last


def check_schedule(plan: dict, num_sms: int, K: int):
    """Assert that the schedule the kernel derives from `plan` computes every
    k-block of every tile exactly once, that each shared tile's contributors
    are the units the kernel will add up, and that partial-sum slots and
    arrival words stay inside the workspace.  Returns the most units sharing
    one tile."""
    tiles = plan["tiles_m"] * plan["tiles_n"]
    num_kb = -(-K // plan["block_k"])
    ctas = plan["cluster_ctas"]
    num_units = plan["grid"] // ctas
    assert plan["grid"] % ctas == 0 and 1 <= num_units <= num_sms // ctas
    full = plan["full_tiles"]
    tail_tiles = tiles - full
    tail_units = plan["tail_units"]
    if tail_tiles == 0:
        assert tail_units == 0 and plan["split"] == 1 and plan["num_slots"] == 0
    else:
        assert tail_tiles <= tail_units <= min(num_units, tail_tiles * num_kb)
        assert full % num_units == 0  # whole rounds before the tail
        assert plan["num_slots"] == tail_units + tail_tiles - 1
    cover = {}
    slots = set()
    for u in range(num_units):
        items = unit_items(u, num_units, full, tail_tiles, tail_units, num_kb)
        assert sum(1 for it in items if it[3] >= 0) <= 2
        for tile, kb0, kb1, r in items:
            assert 0 <= tile < tiles and 0 <= kb0 < kb1 <= num_kb
            cover.setdefault(tile, []).append((kb0, kb1, u))
            if r >= 0:
                first, last = tail_contributors(r, tail_tiles, tail_units, num_kb)
                assert first <= u <= last
                if last > first:
                    slot = u + r
                    assert slot not in slots and 0 <= slot < plan["num_slots"]
                    slots.add(slot)
    # every unit past the last one with work is idle: the grid has none of them
    busy = {u for parts in cover.values() for _, _, u in parts}
    assert busy == set(range(num_units))
    max_parts = 1
    for tile in range(tiles):
        parts = sorted(cover.get(tile, []))
        assert parts, f"tile {tile} is never computed"
        assert parts[0][0] == 0 and parts[-1][1] == num_kb
        for (a0, a1, ua), (b0, b1, ub) in zip(parts, parts[1:]):
            assert a1 == b0 and ub == ua + 1  # consecutive k ranges from consecutive units
        if tile >= full:
            first, last = tail_contributors(tile - full, tail_tiles, tail_units, num_kb)
            assert [u for _, _, u in parts] == list(range(first, last + 1))
        else:
            assert len(parts) == 1
        max_parts = max(max_parts, len(parts))
    assert plan["split"] == max_parts
    return max_parts
