"""Host-side logic of the Python binding: the (layout, leading dimension) it hands the
C ABI for strided torch views, including the single-row/column operands that grouped
calls read in the groups' shared layout. CPU tensors only (no library call)."""
import pytest
import torch

import sm_gemm_b200 as sg


def test_layout_of_plain_and_transposed_views():
    a = torch.zeros(64, 40)
    assert sg._layout(a, "a") == (sg.ROW_MAJOR, 40)
    assert sg._layout(a.t(), "a") == (sg.COL_MAJOR, 40)
    padded = torch.zeros(64, 48)[:, :40]                       # row pitch 48
    assert sg._layout(padded, "a") == (sg.ROW_MAJOR, 48)
    assert sg._layout(padded.t(), "a") == (sg.COL_MAJOR, 48)


def test_layout_rejects_non_unit_strides():
    with pytest.raises(ValueError):
        sg._layout(torch.zeros(8, 8)[::2, ::2], "a")
    with pytest.raises(ValueError):
        sg._layout(torch.zeros(2, 3, 4), "a")


def test_layout_as_reads_single_rows_and_columns_in_either_layout():
    row = torch.zeros(1, 64)                                   # one row, contiguous
    assert sg._layout_as(row, "r", sg.ROW_MAJOR) == (sg.ROW_MAJOR, 64)
    # read as column-major its column pitch is real (1 element); the C ABI rejects that
    # pitch (not 16 bytes), so the binding passes it on rather than inventing another
    assert sg._layout_as(row, "r", sg.COL_MAJOR) == (sg.COL_MAJOR, 1)
    padded_row = torch.zeros(64, 8)[:, :1].t()                 # one row, column pitch 8
    assert sg._layout_as(padded_row, "r", sg.COL_MAJOR) == (sg.COL_MAJOR, 8)
    col = torch.zeros(64, 8)[:, :1]                            # one column of a pitch-8 buffer
    assert sg._layout_as(col, "c", sg.ROW_MAJOR) == (sg.ROW_MAJOR, 8)
    with pytest.raises(ValueError):                            # its 64 elements are 8 apart
        sg._layout_as(col, "c", sg.COL_MAJOR)
    dense_col = torch.zeros(64, 1)                             # 64 consecutive elements
    assert sg._layout_as(dense_col, "c", sg.COL_MAJOR) == (sg.COL_MAJOR, 64)  # unused pitch: >= rows
    with pytest.raises(ValueError):
        sg._layout_as(torch.zeros(4, 8), "x", sg.COL_MAJOR)    # a true row-major matrix
