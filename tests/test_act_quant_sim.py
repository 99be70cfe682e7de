"""The simulated activation-quantisation report runs, and orders the modes as the
element formats imply (E2M1 blocks lose more than E4M3 blocks, both lose something)."""
from tests import act_quant_error as A


def test_act_quant_report_on_the_fixture():
    r = A.simulate("fixture", 32)
    a8, a4 = r["w4a8 (E4M3 blocks)"], r["w4a4 (E2M1 blocks)"]
    assert 0 < a8["rms_err_x_rms"] < a4["rms_err_x_rms"]
    assert 0 < a8["max_err_x_rms"] < a4["max_err_x_rms"]
    # one E4M3 rounding keeps ~2^-4 relative precision per element, so the output's
    # RMS deviation stays well under 25 %, while E2M1 (2^-2) does not stay under 5 %
    assert a8["rms_err_x_rms"] < 0.25 and a4["rms_err_x_rms"] > 0.05
