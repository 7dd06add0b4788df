"""Shared test helpers: moving seeded numpy inputs onto the GPU and back."""
import numpy as np
import torch


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor (bit-identical)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def sample_rows(n_tree: int, n_heads_q: int, count: int, seed: int):
    """(nodes, heads) covering node 0, the last node and random rows."""
    rng = np.random.default_rng(seed)
    nodes = [0, n_tree - 1, n_tree - 1, 0] + list(rng.integers(0, n_tree, size=count))
    heads = [0, n_heads_q - 1, 0, n_heads_q - 1] + list(rng.integers(0, n_heads_q, size=count))
    return np.array(nodes, np.int32), np.array(heads, np.int32)
