"""Developer tool (opt-in pytest plugin): runs the GPU test files against the host build of the
library (build_library.py: the unchanged kernels on the fiber runtime and the device model), to check
the kernels' logic before GPU time is spent on them.  It is not GPU parity: torch's CUDA tensors become
CPU tensors here, and the library the binding loads is replaced by the host build.  Nothing loads it
unless asked:

    python -c "import sys; sys.path.insert(0, 'tests/host_emulation'); import build_library; \
               build_library.build('/tmp/host_lib')"
    MIMO_HOST_LIB=/tmp/host_lib/libmimo_attn_host.so PYTHONPATH=tests/host_emulation \
        python -m pytest -p host_model_plugin tests/test_gpu_bwd.py -m gpu

(cases that need cuBLAS or more than minutes of model time are left out with -k.)
"""
import ctypes
import os

import torch

torch.cuda.is_available = lambda: True
torch.Tensor.cuda = lambda self, *a, **k: self
torch.Tensor.is_cuda = property(lambda self: True)


class _Stream:
    cuda_stream = 0


torch.cuda.current_stream = lambda *a, **k: _Stream()
torch.cuda.synchronize = lambda *a, **k: None
_orig_to = torch.Tensor.to


def _cpu(x):
    if isinstance(x, str) and x.startswith("cuda"):
        return "cpu"
    if isinstance(x, torch.device) and x.type == "cuda":
        return torch.device("cpu")
    return x


def _to(self, *a, **k):
    a = tuple(_cpu(x) for x in a)
    if "device" in k:
        k["device"] = _cpu(k["device"])
    return _orig_to(self, *a, **k)


torch.Tensor.to = _to
_orig_empty, _orig_zeros = torch.empty, torch.zeros


def _dev_kw(f):
    def g(*a, **k):
        if "device" in k:
            k["device"] = _cpu(k["device"])
        return f(*a, **k)
    return g


torch.empty, torch.zeros, torch.arange = _dev_kw(torch.empty), _dev_kw(torch.zeros), _dev_kw(torch.arange)
torch.full, torch.ones = _dev_kw(torch.full), _dev_kw(torch.ones)

from global_attention_moe_b200 import mimo_attn as M  # noqa: E402

_SIM = ctypes.CDLL(os.environ["MIMO_HOST_LIB"])
for name in M.SYMBOLS:
    if hasattr(M.LIB, name) and hasattr(_SIM, name):
        f, rf = getattr(_SIM, name), getattr(M.LIB, name)
        f.argtypes, f.restype = rf.argtypes, rf.restype
M.LIB = _SIM
