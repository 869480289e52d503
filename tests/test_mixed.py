"""Mixed-format fused expert buffers, host side: the layout gives each expert its own
offset by its own format, and the one-stride slicing the page's loader bug used is off by
exactly the factor of two between a packed expert's width and a bf16 expert's."""
import pytest

from fp4_block_scaled_moe_b200.mixed import expert_layout


def test_layout_offsets_follow_each_experts_format():
    rows, K = 1536, 2048
    fmts = ["mxfp4", "bf16", "mxfp4", "mxfp4", "bf16"]
    off, soff, nbytes, sbytes = expert_layout(fmts, rows, K)
    packed, dense = rows * K // 2, rows * 2 * K
    assert off == [0, packed, packed + dense, 2 * packed + dense, 3 * packed + dense]
    assert nbytes == 3 * packed + 2 * dense
    assert soff == [0, rows * K // 32, rows * K // 32, 2 * rows * K // 32, 3 * rows * K // 32]
    assert sbytes == 3 * rows * K // 32
    # every offset is a whole number of packed rows (the unit the kernels address)
    assert all(o % (K // 2) == 0 for o in off)


def test_one_stride_for_all_experts_is_off_by_the_factor_of_two():
    """Sliced with one dtype and one stride, a packed expert's last dimension is half the
    bf16 expert's: 128 against 256 on the same axis for a 256-wide row."""
    K = 256
    packed_width, bf16_width = K // 2, K            # uint8 elements vs bf16 elements per row
    assert (packed_width, bf16_width) == (128, 256) and bf16_width == 2 * packed_width
    rows = 64
    fmts = ["mxfp4", "bf16", "mxfp4"]
    off, _, nbytes, _ = expert_layout(fmts, rows, K)
    uniform = [e * (nbytes // len(fmts)) for e in range(len(fmts))]
    assert uniform != off                            # a single stride misplaces the experts after the bf16 one


def test_unknown_format_is_refused():
    with pytest.raises(ValueError):
        expert_layout(["mxfp4", "fp8"], 64, 256)
