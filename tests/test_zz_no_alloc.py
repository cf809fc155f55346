"""svg_profile_heads_noalloc: profiling for callers that cannot allocate.

Some callers of this library cannot allocate device memory: a plugin inside
an engine that owns all device memory and gives it no workspace, or code in a
region where a cudaMalloc would synchronise the device or is not allowed.
This entry point keeps its scratch in a fixed 16 MiB array owned by the
library.  The GPU test calls it through the C ABI twice in a row and checks
each result against svg_profile_heads (the entry point that takes a
caller-provided workspace), within the tolerance the parity tests use.

The file is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import svg_inputs as si
from sparse_attention_video_svg_b200 import _lib

FAKE = 1 << 20  # 16-byte aligned host value; never dereferenced (rejected on the host)


def test_rejects_shapes_beyond_the_fixed_scratch():
    # 253 heads at d = 128 need 253 * 66560 bytes > 16 MiB per key range
    st = _lib.lib.svg_profile_heads_noalloc(FAKE, FAKE * 2, FAKE * 3, 0, 1, 253, 1024, 128, 4, 256,
                                            1, FAKE * 4, 16, None, FAKE * 5, None)
    assert st == _lib.SVG_ERR_INVALID_ARG
    assert "fixed scratch" in _lib.lib.svg_last_error().decode()


def _run_noalloc(qd, kd, vd, wl, idx_d):
    B, H, N, d = qd.shape
    mse = torch.full((B * H, 2), -1.0, dtype=torch.float32, device=qd.device)
    mode = torch.full((B * H,), -1, dtype=torch.int32, device=qd.device)
    dt = _lib.SVG_BF16 if qd.dtype == torch.bfloat16 else _lib.SVG_FP32
    _lib.call("svg_profile_heads_noalloc", qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), dt, B, H,
              N, d, wl.F, wl.P, wl.width, idx_d.data_ptr(), idx_d.numel(), mse.data_ptr(),
              mode.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return mse.cpu().numpy().astype(np.float64), mode.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [si.WORKLOADS["tiny"], si.small("hunyuan720"),
                                si.WORKLOADS["cogvideox"]], ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point(wl):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_video_svg_b200 as svg
    from tests.helpers import MODE_MARGIN, to_device

    q, k, v, _ = si.generate(wl)
    qd, kd, vd = (to_device(x) for x in (q, k, v))
    idx_d = torch.from_numpy(si.sample_queries(wl)).to("cuda")
    mse_ref, mode_ref = svg.svg_profile_heads(qd, kd, vd, wl.F, wl.P, wl.width, idx_d)
    mse_ref = mse_ref.cpu().numpy().astype(np.float64)
    mode_ref = mode_ref.cpu().numpy()
    if wl.name == "tiny":
        # the small case also straight against the float64 oracle
        from oracle import svg_oracle as O
        mse_o, mode_o = O.profile_heads(*(si.as_float64(x) for x in (q, k, v)),
                                        si.sample_queries(wl), wl.F, wl.P, wl.width)
        mse, mode = _run_noalloc(qd, kd, vd, wl, idx_d)
        for i in range(len(mode_o)):
            for c in range(2):
                assert abs(mse[i, c] - mse_o[i, c]) <= 0.02 * mse_o[i, c] + 2e-5, (i, mse[i], mse_o[i])
            margin = abs(mse_o[i, 0] - mse_o[i, 1]) / max(mse_o[i].max(), 1e-30)
            if margin > MODE_MARGIN:
                assert mode[i] == mode_o[i], i
    for call in range(2):
        mse, mode = _run_noalloc(qd, kd, vd, wl, idx_d)
        for i in range(len(mode_ref)):
            for c in range(2):
                r = mse_ref[i, c]
                assert abs(mse[i, c] - r) <= 0.02 * r + 2e-5, (wl.name, call, i, mse[i], mse_ref[i])
            margin = abs(mse_ref[i, 0] - mse_ref[i, 1]) / max(mse_ref[i].max(), 1e-30)
            if margin > MODE_MARGIN:
                assert mode[i] == mode_ref[i], (wl.name, call, i)
