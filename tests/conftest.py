import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 GPU (sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


# Collection order for a run that stops at the first failure (-x): the parity
# tests of the training step, its kernels and decode first, then the
# allocation-free entry (its file sets up per-device state on first use, which
# no other test reads), and last the tests of the entry points built on the
# step, in this order: L-infinity clipping, data parallelism, the C program,
# resume, the extended sampler, longer contexts, the configuration limits,
# dropout.
_NEXT = ("test_zz_no_alloc.py",)
_LATE = ("test_gpu_clip_linf.py", "test_gpu_dp.py", "test_gpu_c_abi.py", "test_gpu_resume.py",
         "test_gpu_sample_ext.py", "test_gpu_long_context.py", "test_gpu_limits.py",
         "test_gpu_dropout.py")


def pytest_collection_modifyitems(session, config, items):
    def rank(item):
        name = os.path.basename(str(item.fspath))
        if name in _LATE:
            return 2 + _LATE.index(name)
        return 1 if name in _NEXT else 0
    items.sort(key=rank)  # stable: the order inside each group is kept
