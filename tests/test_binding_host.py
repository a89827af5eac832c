"""Host logic of the Python binding on CPU (no kernel runs): which tensors the wrappers pass to the
strided entry points and with which thrift_strides."""

import pytest
import torch

from precision_attention_block_b200 import _strides


def test_dense_tensors_need_no_strides():
    assert _strides(None) is None
    assert _strides(torch.zeros(2, 4, 16, 8, dtype=torch.float16)) is None


def test_token_major_view():
    """A [B, N, H, d] tensor seen as [B, H, N, d]: batch stride N*H*d, head stride d, token stride H*d."""
    B, N, H, d = 2, 16, 4, 8
    x = torch.zeros(B, N, H, d, dtype=torch.float16).transpose(1, 2)
    st = _strides(x)
    assert (st.b, st.h, st.n) == (N * H * d, d, H * d)


def test_padded_rows_view():
    x = torch.zeros(2, 2, 16, 72, dtype=torch.float16)[..., :64]
    st = _strides(x)
    assert (st.b, st.h, st.n) == (2 * 16 * 72, 16 * 72, 72)


def test_non_unit_channel_stride_is_refused():
    x = torch.zeros(1, 2, 8, 16, dtype=torch.float16).transpose(2, 3)
    with pytest.raises(ValueError):
        _strides(x)
    with pytest.raises(ValueError):
        _strides(torch.zeros(4, 8, 16, dtype=torch.float16)[:, ::2])


def test_strides_of_size_one_dimensions_are_the_dense_ones():
    """torch may report any stride for a dimension of size 1; it is never used, so the dense
    layout's stride (a valid multiple of 16 bytes) is passed instead."""
    x = torch.zeros(1, 16, 4, 8, dtype=torch.float16).transpose(1, 2)
    assert _strides(x).b == 4 * 16 * 8
    y = torch.zeros(3, 16, 1, 8, dtype=torch.float16).transpose(1, 2)[:, :, ::2]
    st = _strides(y)
    assert (st.b, st.h, st.n) == (16 * 8, 8 * 8, 16)
