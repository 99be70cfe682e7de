"""The tensor-core rate probe (the separate measurement library): it runs on
the device and reports plausible rates. A sanity check of the tool, kept out of
the parity tests: it asserts no speed, only that each rate is positive and no
higher than the UMMA kind can physically issue (the nominal dense rate per SM
clock, with a margin for clock readings)."""
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_moe_layer_05_b200 import build
    build.build()


@pytest.mark.parametrize("kind,nominal", [(0, 4096), (1, 8192), (2, 16384)],
                         ids=["bf16", "e2m1_x_e4m3", "e2m1_x_e2m1"])
def test_tensor_rate_probe_reports_a_plausible_rate(kind, nominal):
    from sparse_moe_layer_05_b200 import binding as B
    r = B.moe_probe_tensor_rate(kind, 256, 16)
    print(f"[probe] kind {kind}: {r:.0f} MAC per SM clock (nominal dense {nominal})")
    assert 0 < r <= 1.1 * nominal, r
