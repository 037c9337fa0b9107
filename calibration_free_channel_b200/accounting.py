"""Read accounting in 32-byte sectors.

The pages count reads the way the GPU bills them: a 32-byte sector touched at
all counts in full ("KAIST: MoE Decoding Needs No Calibration Data", section
"Calibrated thresholds do not pin down how much you read").  For one MoE block
step, every active expert is charged once per step (its sketch, the union of
its tokens' candidate rows, the union of their kept down rows and its
low-rank map), plus the router.

Every row the reader touches starts on a 32-byte boundary and is a multiple
of 32 bytes long (gate/up/down rows are 2d bytes, sketch rows d/4 bytes,
alpha blocks 4I bytes, low-rank rows 2r bytes with r % 16 == 0 or whole
blocks; base-3 sketch rows are padded to whole sectors), so the sector count
times 32 equals the byte count.
"""
from __future__ import annotations

import numpy as np

SECTOR = 32


def expert_bytes(I: int, d: int, r: int, n_cand_rows: int, n_kept_rows: int, packing: str = "2bit") -> dict:
    """Algorithmic bytes of one active expert in one step."""
    sketch = 2 * I * sketch_row_bytes(d, packing) + 2 * I * 4
    cand = 2 * n_cand_rows * d * 2
    down = n_kept_rows * d * 2
    lowrank = (I + d) * r * 2 if r > 0 else 0
    return dict(sketch=sketch, cand=cand, down=down, lowrank=lowrank,
                total=sketch + cand + down + lowrank)


def sketch_row_bytes(d: int, packing: str = "2bit") -> int:
    """Bytes of one resident sketch row: 2-bit codes (d / 4), or base 3 with
    five trits per byte, ceil(d / 5) bytes rounded up to whole sectors."""
    if packing == "2bit":
        return d // 4
    if packing == "base3":
        return -(-((d + 4) // 5) // SECTOR) * SECTOR
    raise ValueError(packing)


def sketch_footprint(I: int, d: int, packing: str = "2bit") -> float:
    """Resident sketch of one expert (gate and up rows plus alpha) as a
    fraction of its BF16 gate, up and down weights."""
    return (2 * I * sketch_row_bytes(d, packing) + 2 * I * 4) / dense_expert_bytes(I, d)


def dense_expert_bytes(I: int, d: int) -> int:
    return 3 * I * d * 2


def router_bytes(E: int, d: int, bias: bool) -> int:
    return E * d * 2 + (E * 4 if bias else 0)


def step_bytes(E: int, I: int, d: int, r: int, ids: np.ndarray, cand: np.ndarray, kept: np.ndarray,
               bias: bool = False, packing: str = "2bit") -> dict:
    """Bytes of one sparse step over B tokens.

    ids [B, top_e] routed experts; cand [B, top_e, c] and kept [B, top_e, k]
    channel indices per (token, slot).  Rows are counted over the union of the
    tokens routed to each expert."""
    ids = np.asarray(ids)
    per = {}
    for e in np.unique(ids):
        bs, ss = np.nonzero(ids == e)
        cu = np.unique(np.concatenate([np.asarray(cand)[b, s] for b, s in zip(bs, ss)]))
        ku = np.unique(np.concatenate([np.asarray(kept)[b, s] for b, s in zip(bs, ss)]))
        per[int(e)] = expert_bytes(I, d, r, cu.size, ku.size, packing)
    total = router_bytes(E, d, bias) + sum(v["total"] for v in per.values())
    return dict(per_expert=per, router=router_bytes(E, d, bias), total=total,
                dense=router_bytes(E, d, bias) + len(per) * dense_expert_bytes(I, d))


def fixed_budget_step_bytes(E: int, I: int, d: int, r: int, k: int, c: int, n_experts: int,
                            bias: bool = False) -> int:
    """Bytes of a step whose tokens share no expert (exactly B*top_e active
    (token, expert) pairs, or one token): each pair reads c candidate rows and
    k down rows.  Top-k fixes this count whatever the input."""
    return router_bytes(E, d, bias) + n_experts * expert_bytes(I, d, r, c, k)["total"]
