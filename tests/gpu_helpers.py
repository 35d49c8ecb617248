"""Helpers shared by the GPU parity tests: host<->device moves and by-row state comparison."""
import numpy as np
import torch

DEV = "cuda:0"


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> bf16 device tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def i32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a), dtype=np.int32)).to(DEV)


def u32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.uint32)).view(np.int32)).to(DEV)


def f32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def mask_host(mask):
    """Host snapshot of a binding.Mask."""
    c = host(mask.counts)
    return dict(
        charge=host(mask.charge),
        words=host(mask.words).view(np.uint32),
        rows=host(mask.active_rows)[: c[0]],
        tiles=host(mask.active_tiles)[: c[1]],
        tile_rows=host(mask.tile_rows)[: c[1]],
        counts=c,
        row_slot=host(mask.row_slot),
        slot_step=host(mask.slot_step),
        free=host(mask.free_slots),
    )


def check_slot_invariants(mh, slot_cap):
    """Every active row holds a distinct slot (or none after overflow); nothing else holds one.
    Also: tile_rows[j] is the position in active_rows of the first row of the j-th active tile."""
    R = mh["row_slot"].size
    for j, w in enumerate(mh["tiles"]):
        assert mh["rows"][mh["tile_rows"][j]] // 32 == w
        assert mh["tile_rows"][j] == 0 or mh["rows"][mh["tile_rows"][j] - 1] // 32 < w
    active = np.zeros(R, bool)
    active[mh["rows"]] = True
    slots = mh["row_slot"]
    assert np.all(slots[~active] == -1)
    held = slots[active & (slots >= 0)]
    assert len(np.unique(held)) == len(held)
    assert np.all((held >= 0) & (held < slot_cap))
    n_without = int(np.sum(active & (slots < 0)))
    assert mh["counts"][3] == n_without
    assert mh["counts"][2] == slot_cap - len(held)
    free = mh["free"][: mh["counts"][2]]
    assert len(np.intersect1d(free, held)) == 0


def rel_err(got: np.ndarray, ref: np.ndarray, floor_frac: float = 1e-3) -> float:
    """max |got - ref| / max(|ref|, floor_frac * max|ref|)."""
    ref = ref.astype(np.float64)
    floor = floor_frac * max(np.abs(ref).max(), 1e-30)
    return float(np.max(np.abs(got.astype(np.float64) - ref) / np.maximum(np.abs(ref), floor)))
