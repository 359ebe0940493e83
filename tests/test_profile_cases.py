"""The profiling-case module (what the committed ncu commands run): its case
table and its command-line checks, without a GPU."""
import pytest

from causal_linear_attention_chunked_b200 import profile_cases


def test_cases_listed():
    assert set(profile_cases.CASES) == {"fused", "decode", "bwd", "gqa"}
    assert all(callable(f) for f in profile_cases.CASES.values())


@pytest.mark.parametrize("argv", [[], ["nope"], ["fused", "decode"]])
def test_bad_arguments_exit_with_usage(argv):
    with pytest.raises(SystemExit) as e:
        profile_cases.main(argv)
    assert "usage" in str(e.value)
