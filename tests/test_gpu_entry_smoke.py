"""The package entry point's smoke check (one small bf16 step on cuda:0, its P,
loss and dL against the float64 oracle) runs here as a GPU test as well."""
import pytest

pytestmark = pytest.mark.gpu


def test_entry_point_smoke(gpu_lib, capsys):
    import __graft_entry__ as entry

    entry.smoke()
    assert "smoke ok" in capsys.readouterr().out
