"""ttq_act_stats_noalloc, the allocation-free statistic entry point.

Some callers cannot allocate device memory (cudaMalloc can stall the whole device, and
some host programs have handed every byte of HBM to their own allocator), so this entry
point keeps its reduction scratch in a fixed array inside the library instead of a
caller workspace. It must give the same s as ttq_act_stats, call after call, since
every call reuses (and must re-clear) the same array. This file is collected last.
"""

import ctypes

import numpy as np
import pytest

import online_activation_aware_b200 as ttq

TOO_LARGE = -7


def _stream(torch):
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_noalloc_rejects_oversized_d_without_launching():
    lib = ttq.load_library()
    a = ctypes.c_void_p(1 << 20)  # fake aligned address: the size check comes first
    rc = lib.ttq_act_stats_noalloc(a, 16, 65544, 65544, ctypes.c_float(0.5), ctypes.c_float(0.4), 2, a, None)
    assert rc == TOO_LARGE
    assert lib.ttq_status_string(TOO_LARGE).decode() == "TTQ_ERR_TOO_LARGE"


@pytest.mark.gpu
@pytest.mark.parametrize("T,d,ld_x,p", [(3000, 5120, 5120, 2), (17, 264, 264, 2), (4096, 2048, 2048, 1),
                                        (600, 65536, 65536, 2), (4096, 776, 784, 2)])
def test_noalloc_matches_workspace_entry_point_twice(T, d, ld_x, p):
    # (4096, 776, 784): rows wider than d and a last column strip of 8 channels, with the
    # rows split over many blocks, so the arrival counters meet a partial strip
    torch = pytest.importorskip("torch")
    from online_activation_aware_b200 import synthetic
    from oracle import ttq_oracle as O

    lib = ttq.load_library()
    Xh = synthetic.as_bf16(synthetic.draw_layer(T, d, 8, seed=T + d)[0])
    wide = torch.zeros(T, ld_x, dtype=torch.bfloat16)
    wide[:, :d] = Xh
    wide[:, d:] = 1.0e4  # padding past d must not count
    X = wide.cuda()
    ref = ttq.act_stats(Xh.cuda(), 0.5, 0.4, p).cpu().numpy()
    s64, _ = O.act_stats(synthetic.bf16_values(Xh), 0.5, 0.4, p)
    for _ in range(2):  # two calls in a row: the shared scratch must be re-cleared
        s = torch.full((d,), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.ttq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), T, d, ld_x, ctypes.c_float(0.5),
                                       ctypes.c_float(0.4), p, ctypes.c_void_p(s.data_ptr()), _stream(torch))
        assert rc == 0
        torch.cuda.synchronize()
        got = s.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref) / ref) <= 1e-5
        assert np.max(np.abs(got.astype(np.float64) - s64) / s64) <= 1e-5
    assert ttq.device_status() == 0
