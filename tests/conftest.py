import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case that takes tens of seconds")


def golden_path(name: str) -> str:
    return os.path.join(ROOT, "tests", "golden", name)


def read_golden(name: str):
    """Rows of a whitespace-separated fixture, skipping '#' comment lines."""
    rows = []
    with open(golden_path(name), encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ------------------------------------------------------------ GPU helpers
def to_device_bf16(a, device="cuda"):
    """numpy uint16 bf16 patterns -> torch bf16 tensor on the device (same bytes)."""
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def to_host_u16(t):
    import numpy as np
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_tensor_to_f64(t):
    import numpy as np
    return ((to_host_u16(t).astype(np.uint32) << 16).view(np.float32)).astype(np.float64)


def canary_buffer(nbytes, margin=4096, device="cuda"):
    """A uint8 buffer filled with 0xCD and a view of nbytes in its middle
    (16-byte aligned); check_canary() verifies the margins are untouched."""
    import torch
    buf = torch.full((nbytes + 2 * margin,), 0xCD, dtype=torch.uint8, device=device)
    return buf, buf[margin: margin + nbytes]


def check_canary(buf, nbytes, margin=4096):
    import torch
    head = buf[:margin]
    tail = buf[margin + nbytes:]
    assert bool(torch.all(head == 0xCD)) and bool(torch.all(tail == 0xCD)), "write outside the output buffer"
