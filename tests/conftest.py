import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


# Suites that run after all others, in this order, so that a run stopping at its first failure has
# already run the main forward-path suites: the prefill shapes with a single value slot, the window
# and bias extension, landmark generation (a step before the forward path), the debug check of a
# caller's selection, the backward pass, and last of all the allocation-free entry point (its first
# call sets up a per-device array), so that every other test has run before it.
RUN_LAST = ("test_parity_one_value_slot.py", "test_parity_window.py", "test_parity_landmarks.py",
            "test_check_selection.py", "test_parity_backward.py", "test_zz_no_alloc.py")


def pytest_collection_modifyitems(config, items):
    def order(item):
        name = os.path.basename(str(item.fspath))
        return RUN_LAST.index(name) + 1 if name in RUN_LAST else 0
    items.sort(key=order)
