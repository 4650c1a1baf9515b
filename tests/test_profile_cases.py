"""Host-side checks of the profiling driver (no GPU needed)."""
import pytest

from block_causal_attention_dit_b200 import profile_cases


def test_usage_without_arguments(capsys):
    assert profile_cases.main([]) == 2
    assert "cases" in capsys.readouterr().out


def test_unknown_case_is_rejected_before_any_device_work():
    with pytest.raises(ValueError):
        profile_cases.run("nope", 1, 1)
