"""options_from_config: the fixed-buffer keys of a DeepSpeed-style config
("ZeRO：从优化器状态到残差状态的显存优化" section 3.3 "CB") mapped onto
ZeroOptimizer's keyword arguments.  Host only."""
import inspect

import pytest


def _z():
    import zero_sharded_optimizer_sm_b200 as z

    return z


def test_the_pages_snippet():
    z = _z()
    cfg = {"communication_data_type": "fp16", "allgather_bucket_size": 200000000,
           "reduce_bucket_size": 200000000}
    assert z.options_from_config(cfg) == {"bucket_elems": 200000000, "dtype": z.ZERO_DTYPE_F16}


def test_nested_zero_optimization_section_and_stage():
    z = _z()
    cfg = {"bf16": {"enabled": True}, "communication_data_type": "bf16",
           "zero_optimization": {"stage": 3, "reduce_bucket_size": 5e8, "allgather_bucket_size": 5e8,
                                 "overlap_comm": True}}
    assert z.options_from_config(cfg) == {"stage": 3, "bucket_elems": 500000000, "dtype": z.ZERO_DTYPE_BF16}


def test_bucket_rounded_up_to_the_granule_and_either_key_alone():
    z = _z()
    assert z.options_from_config({"reduce_bucket_size": 1001}) == {"bucket_elems": 1008}
    assert z.options_from_config({"allgather_bucket_size": 64}) == {"bucket_elems": 64}
    assert z.options_from_config({}) == {}


@pytest.mark.parametrize("cfg", [
    {"reduce_bucket_size": 200, "allgather_bucket_size": 400},  # two buckets: the fused step has one
    {"communication_data_type": "fp32"},
    {"zero_optimization": {"stage": 0}},
    {"stage": 4},
    {"reduce_bucket_size": 0},
])
def test_what_cannot_be_honoured_raises(cfg):
    with pytest.raises(ValueError):
        _z().options_from_config(cfg)


def test_the_result_is_valid_keyword_arguments_of_zero_optimizer():
    z = _z()
    params = inspect.signature(z.ZeroOptimizer.__init__).parameters
    out = z.options_from_config({"communication_data_type": "fp16", "reduce_bucket_size": 1 << 20,
                                 "zero_optimization": {"stage": 2}})
    assert set(out) <= set(params), set(out) - set(params)
