import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 GPU (sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


# Collection order for a run that stops at the first failure (-x): the parity
# tests of the training step, its kernels and decode first, then the tests of
# the entry points built on the step, in this order: L-infinity clipping, data
# parallelism (against itself, then against the oracle), the C program,
# resume, the extended sampler, longer contexts, the configuration limits,
# dropout; the allocation-free entry's file is collected last of all, so a
# failure there stops nothing else.
_LATE = ("test_gpu_clip_linf.py", "test_gpu_dp.py", "test_gpu_dp_oracle.py", "test_gpu_c_abi.py",
         "test_gpu_resume.py", "test_gpu_sample_ext.py", "test_gpu_long_context.py",
         "test_gpu_limits.py", "test_gpu_dropout.py")
_LAST = ("test_zz_no_alloc.py",)


def pytest_collection_modifyitems(session, config, items):
    def rank(item):
        name = os.path.basename(str(item.fspath))
        if name in _LAST:
            return 1 + len(_LATE)
        if name in _LATE:
            return 1 + _LATE.index(name)
        return 0
    items.sort(key=rank)  # stable: the order inside each group is kept
