"""The bounded-wait path on the GPU without a fault: a wait on an mbarrier that nothing
arrives on gives up after its limit, the device error word says SFM_ERR_TIMEOUT, the
context stays usable and the next kernels run normally."""
import ctypes

import pytest
import torch

from selective_scan_sfm_b200 import _abi, sfm_get_device_error, sfm_selective_scan_fold, synth

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports_timeout():
    sfm_get_device_error(clear=True)
    s = torch.cuda.current_stream()
    rc = _abi.lib().sfm_selftest_wait_timeout(20000, ctypes.c_void_p(s.cuda_stream))  # 20 ms
    assert rc == _abi.SFM_OK
    assert sfm_get_device_error(clear=True) == _abi.SFM_ERR_TIMEOUT
    assert sfm_get_device_error(clear=True) == _abi.SFM_OK  # cleared
    # the context is intact: a forward runs and reports no error
    d = synth.make_inputs(B=2, D=32, T=20, N=8, dtype="f32", seed=1)
    dc = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    y = sfm_selective_scan_fold(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], z=dc["z"], conv_w=dc["conv_w"],
                                conv_b=dc["conv_b"], aux_init=True)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    assert sfm_get_device_error(clear=True) == _abi.SFM_OK
