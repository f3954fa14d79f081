"""Host-side argument marshalling of the Python binding, on CPU: the (B, D)
row operands' pointer and batch stride, and the errors for layouts the
library does not take.  The CUDA-device check is stubbed out so that CPU
tensors stand in for device ones; nothing reaches the library."""
import pytest
import torch

from scan_gated_rnns_b200 import ops


@pytest.fixture(autouse=True)
def _cpu_tensors(monkeypatch):
    monkeypatch.setattr(ops, "_need_cuda", lambda t, name: None)


def test_rows_pointer_and_batch_stride():
    like = torch.zeros(4, 8)
    assert ops._rows(None, 4, 8, like, "h0") == (0, 0)
    t = torch.randn(4, 8)
    assert ops._rows(t, 4, 8, like, "h0") == (t.data_ptr(), 8)
    # a time row of a (B, T, D) tensor: batch stride T * D
    seq = torch.randn(4, 5, 8)
    row = seq[:, 2, :]
    assert ops._rows(row, 4, 8, like, "k_t") == (row.data_ptr(), 5 * 8)
    # one batch row: the stride is not used, D is passed
    one = torch.randn(3, 8)[1:2]
    assert ops._rows(one, 1, 8, like[:1], "h0") == (one.data_ptr(), 8)
    # a (D,) vector: one state shared by every batch row (stride 0)
    v = torch.randn(8)
    assert ops._rows(v, 4, 8, like, "h0") == (v.data_ptr(), 0)
    # D = 1: any stride along D is accepted
    col = torch.randn(4, 3)[:, 1:2]
    assert ops._rows(col, 4, 1, torch.zeros(4, 1), "h0") == (col.data_ptr(), 3)


@pytest.mark.parametrize("bad,msg", [
    (lambda: torch.randn(4, 8, dtype=torch.float64), "dtype"),
    (lambda: torch.randn(8, 4).t(), "contiguous along D"),
    (lambda: torch.randn(4, 9), r"\(B, D\)"),
    (lambda: torch.randn(5, 8), r"\(B, D\)"),
    (lambda: torch.randn(4, 8, 1), r"\(B, D\)"),
    (lambda: torch.randn(9), r"\(D,\) vector"),
    (lambda: torch.randn(16)[::2], r"\(D,\) vector"),
])
def test_rows_refuses_other_layouts(bad, msg):
    with pytest.raises(ValueError, match=msg):
        ops._rows(bad(), 4, 8, torch.zeros(4, 8), "h0")
