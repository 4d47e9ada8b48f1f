"""Host <-> device marshalling for the GPU parity tests (no arithmetic here)."""

import numpy as np
import torch

DEV = "cuda:0"


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def dev_f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).to(DEV)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def status_word() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def sample_rows(M: int, tile: int = 128):
    """Rows that touch every M tile: the first and last row of each tile and the ragged tail."""
    rows = set()
    for t0 in range(0, M, tile):
        rows.update({t0, min(M - 1, t0 + tile - 1), min(M - 1, t0 + 37)})
    rows.add(M - 1)
    return sorted(rows)
