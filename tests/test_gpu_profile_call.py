"""The one-call profiling runner runs the path on a named workload."""
import pytest

pytestmark = pytest.mark.gpu


def test_profile_call_tiny(capsys):
    from video_dit_sparse_da2_b200 import profile_call
    profile_call.main(["tiny"])
    assert capsys.readouterr().out.strip().endswith("ok")


def test_profile_call_fewer_heads(capsys):
    from video_dit_sparse_da2_b200 import profile_call
    profile_call.main(["tiny", "--heads", "1"])
    assert capsys.readouterr().out.strip().endswith("ok")
