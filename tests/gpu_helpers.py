"""Small helpers shared by the GPU parity tests (no arithmetic of the method)."""
import numpy as np
import torch

DEV = "cuda:0"


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    """fp32 array of bf16-representable values -> bf16 CUDA tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV).to(torch.bfloat16).contiguous()


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV).contiguous()


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def host_bytes(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.uint8).cpu().numpy().reshape(-1)


def check_status(status: torch.Tensor) -> int:
    torch.cuda.synchronize()
    return int(status.item())
