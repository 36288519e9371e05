"""Test helpers: host/device transfer of bit patterns and the MMA scale layout
index map as include/nvfp4moe.h defines it. No quantization arithmetic."""
import numpy as np
import torch


def dev_bf16(bits: np.ndarray, dev) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.to(dev).view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def dev_u8(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(dev)


def dev_f32(a, dev) -> torch.Tensor:
    return torch.as_tensor(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def mma_index(rows: int, nsc: int) -> np.ndarray:
    """idx[r, c] = byte offset of scale (r, c) in the MMA layout."""
    r = np.arange(rows)[:, None]
    c = np.arange(nsc)[None, :]
    chunk = (r // 128) * (nsc // 4) + c // 4
    return chunk * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)


def mma_rows_to_rowmajor(flat: np.ndarray, rows_idx: np.ndarray, nsc: int) -> np.ndarray:
    """Row-major scales of the listed rows of an MMA-layout scale buffer."""
    r = np.asarray(rows_idx, np.int64)[:, None]
    c = np.arange(nsc)[None, :]
    chunk = (r // 128) * (nsc // 4) + c // 4
    return np.asarray(flat).reshape(-1)[chunk * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)]


def mma_to_rowmajor(flat: np.ndarray, rows: int, nsc: int) -> np.ndarray:
    return np.asarray(flat).reshape(-1)[mma_index(rows, nsc)]


def rowmajor_to_mma(sc: np.ndarray) -> np.ndarray:
    rows, nsc = sc.shape
    out = np.zeros(rows * nsc, np.uint8)
    out[mma_index(rows, nsc)] = sc
    return out


def sync():
    torch.cuda.synchronize()
