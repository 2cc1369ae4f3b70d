"""The fused kernel's bounded waits on other CTAs, made to run out on purpose.

``ssd_fwd_withhold_publish`` runs the forward with one chunk owner that never
publishes its state and a short bound on every wait for another CTA's flag.
The blocks that need that state give up, the status word reads
SSD_ERR_TIMEOUT, the kernel still finishes, and the device stays usable: a
normal call right after matches the oracle.  Nothing here faults or hangs the
GPU: the flag is simply never set, and the waits are bounded.
"""
import ctypes

import pytest
import torch

import oracle
from parity import assert_close
from structured_state_space_ssd_b200 import make_inputs
from structured_state_space_ssd_b200 import ssd as S

pytestmark = pytest.mark.gpu

SSD_ERR_TIMEOUT = 4


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("shape,withhold", [
    ((2, 768, 4, 64, 128, 1, 256), (0, 0, 0)),
    ((2, 768, 4, 64, 128, 1, 256), (1, 3, 1)),
    ((1, 8448, 2, 64, 128, 1, 256), (0, 1, 5)),   # 33 chunks: look-back finds neither S~_5 nor L_5
])
def test_a_withheld_state_times_out_and_the_device_stays_usable(shape, withhold, cuda_device):
    batch, T, H, P, N, G, Q = shape
    inp = make_inputs(batch, T, H, P, N, G, "bf16", seed=41, with_init=True)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    lib = S.load()
    code = S.SSD_BF16
    ws = torch.empty(S.ssd_fwd_workspace_bytes(batch, T, H, P, G, N, Q, code), dtype=torch.uint8,
                     device=cuda_device)
    y = torch.empty_like(d["x"])
    fin = torch.empty((batch, H, P, N), dtype=torch.float32, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device)
    wb, wh, wc = withhold
    rc = lib.ssd_fwd_withhold_publish(
        _p(d["x"]), _p(d["dt"]), _p(d["A"]), _p(d["B"]), _p(d["C"]), _p(d["D"]), Q, _p(d["init_state"]), _p(y),
        _p(fin), batch, T, H, P, G, N, code, _p(ws), ctypes.c_size_t(ws.numel()),
        ctypes.c_void_p(stream.cuda_stream), wb, wh, wc, 20000)
    assert rc == 0, S.status_string(rc)
    assert S.ssd_fwd_check(ws, stream) == SSD_ERR_TIMEOUT
    torch.cuda.synchronize(cuda_device)  # the stream completed: the kernel returned
    # the same workspace and device serve a normal call afterwards
    y2, fin2 = S.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], Q, d["init_state"], workspace=ws)
    assert S.ssd_fwd_check(ws, stream) == 0
    y_ref, fin_ref = oracle.ssd_ref_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                        init_state=inp["init_state"])
    assert_close(y2.float().cpu().numpy(), y_ref, "bf16", "y after the timed-out call")
    assert_close(fin2.cpu().numpy(), fin_ref, "bf16", "final_state after the timed-out call")


def test_withhold_hook_validates_its_arguments(cuda_device):
    lib = S.load()
    inp = make_inputs(1, 512, 2, 64, 64, 1, "bf16", seed=2)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    ws = torch.empty(S.ssd_fwd_workspace_bytes(1, 512, 2, 64, 1, 64, 256, S.SSD_BF16), dtype=torch.uint8,
                     device=cuda_device)
    y = torch.empty_like(d["x"])
    args = (_p(d["x"]), _p(d["dt"]), _p(d["A"]), _p(d["B"]), _p(d["C"]), _p(d["D"]), 256, None, _p(y), None,
            1, 512, 2, 64, 1, 64, S.SSD_BF16, _p(ws), ctypes.c_size_t(ws.numel()), None)
    assert lib.ssd_fwd_withhold_publish(*args, 1, 0, 0, 100) == 1   # batch index out of range
    assert lib.ssd_fwd_withhold_publish(*args, 0, 2, 0, 100) == 1   # head index out of range
    assert lib.ssd_fwd_withhold_publish(*args, 0, 0, 0, 0) == 1     # no poll bound
    # a problem on the CUDA-core path has no such hand-off
    f32 = make_inputs(1, 256, 2, 16, 16, 1, "f32", seed=3)
    e = {k: (v.to(cuda_device) if v is not None else None) for k, v in f32.items()}
    y32 = torch.empty_like(e["x"])
    ws32 = torch.empty(S.ssd_fwd_workspace_bytes(1, 256, 2, 16, 1, 16, 64, S.SSD_F32), dtype=torch.uint8,
                       device=cuda_device)
    rc = lib.ssd_fwd_withhold_publish(_p(e["x"]), _p(e["dt"]), _p(e["A"]), _p(e["B"]), _p(e["C"]), _p(e["D"]), 64,
                                      None, _p(y32), None, 1, 256, 2, 16, 1, 16, S.SSD_F32, _p(ws32),
                                      ctypes.c_size_t(ws32.numel()), None, 0, 0, 0, 100)
    assert rc == 2
