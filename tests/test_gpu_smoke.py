"""The smoke entry point (`__graft_entry__.smoke`) as a GPU test, so that a
change of kernel choice or numerics that breaks it shows in the suite."""
import os
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def test_smoke_runs():
    import __graft_entry__
    __graft_entry__.smoke()
