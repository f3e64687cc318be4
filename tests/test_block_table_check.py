"""The binding's optional host-side block-table check (debugging aid; the
kernels do not validate block ids, as the operator documentation states)."""
import pytest
import torch

import workloads as W
from paged_attention_02_b200 import validate_block_tables


def _problem(layout=0):
    return W.make_problem(seed=3, seq_len=[1, 1, 2], kv_seq_len=[33, 16, 70], head_num=4,
                          kv_head_num=2, head_size=64, block_size=16, spare_blocks=3,
                          pad_value=-1, kv_layout=layout)


@pytest.mark.parametrize("layout", [0, 1])
def test_valid_tables_pass_and_padding_is_ignored(layout):
    p = _problem(layout)
    validate_block_tables(p.block_tables, p.kv_seq_len, p.block_size, p.key_cache.shape[0])
    bt = p.block_tables.clone()
    bt[0, 3:] = 10 ** 6                     # past ceil(33 / 16) = 3: never read
    validate_block_tables(bt, p.kv_seq_len, p.block_size, p.key_cache.shape[0])


@pytest.mark.parametrize("value", [-1, "num_blocks", 2 ** 30])
def test_out_of_range_entry_in_the_read_range_is_reported(value):
    p = _problem()
    nb = p.key_cache.shape[0]
    bt = p.block_tables.clone()
    bt[2, 4] = nb if value == "num_blocks" else value    # ceil(70 / 16) = 5 entries read
    with pytest.raises(ValueError, match=r"block_tables\[2\]\[4\]"):
        validate_block_tables(bt, p.kv_seq_len, p.block_size, nb)


def test_short_table_row_is_reported():
    p = _problem()
    bt = p.block_tables[:, :2].contiguous()
    with pytest.raises(ValueError, match="needs 3 blocks"):
        validate_block_tables(bt, p.kv_seq_len, p.block_size, p.key_cache.shape[0])


def test_fiaop_runs_the_check_before_planning():
    """With check_block_tables=True a bad entry is reported before phase 1
    (so this runs without a GPU)."""
    from paged_attention_02_b200 import FiaOp
    p = _problem()
    bt = p.block_tables.clone()
    bt[1, 0] = -5
    with pytest.raises(ValueError, match=r"block_tables\[1\]\[0\]"):
        FiaOp(p.query, p.key_cache, p.value_cache, bt, [int(x) for x in p.seq_len],
              [int(x) for x in p.kv_seq_len], p.head_num, p.kv_head_num, p.qk_scale,
              check_block_tables=True)
