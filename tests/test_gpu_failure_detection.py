"""The failure-detection path on the GPU, exercised without a fault (B200).

Every hand-off between the warps of a libtq kernel is an mbarrier wait bounded in time; a wait that
runs out records a code in the library's device error word and the kernel returns. tq_selftest_wait
runs that wait on an mbarrier nothing arrives on (1 ms limit): tq_sync_check must then report
TQ_ERR_DEVICE_TIMEOUT once, clear it, and the next library call must work and match the oracle.
"""
import math

import numpy as np
import pytest

import workloads as W
from oracle import attention as OA
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import normwise_rel, np_f16, np_u32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def test_timeout_is_reported_once_and_cleared(dev):
    tq.tq_sync_check()                                   # nothing pending
    tq.tq_selftest_wait(1_000_000)
    with pytest.raises(tq.TQError) as e:
        tq.tq_sync_check()
    assert e.value.status == tq.TQ_ERR_DEVICE_TIMEOUT
    tq.tq_sync_check()                                   # cleared
    # the context is still usable: an encode + attention step afterwards matches the oracle
    d, T, Hq = 128, 700, 4
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    K = W.kv_slice(T, d, 3, 20.0, 0.5, 0, W.TAG_K, 9, 0)
    V = W.kv_slice(T, d, 3, 20.0, 0.5, 0, W.TAG_V, 9, 0)
    cbk, cbv = tq.tq_codebook_init(d, 3), tq.tq_codebook_init(d, 1)
    kc, kn = tq.empty_mse(T, d, 3)
    vc, vs, vn, vg = tq.empty_prod(T, d, 2)
    tq.tq_encode_mse(cbk, torch.from_numpy(K).to(dev).to(torch.bfloat16), rot, kc, kn)
    tq.tq_encode_prod(cbv, torch.from_numpy(V).to(dev).to(torch.bfloat16), rot, vc, vs, vn, vg)
    q_np = W.queries_bf16((1, Hq, d))
    out = torch.empty((1, Hq, d), dtype=torch.float32, device=dev)
    tq.tq_attend_decode(cbk, cbv, torch.from_numpy(q_np).to(dev).to(torch.bfloat16), rot, kc, kn.view(1, 1, T), vc,
                        vn.view(1, 1, T), out, v_signs=vs, v_gammas=vg.view(1, 1, T))
    tq.tq_sync_check()
    kh = Q.decode(np_u32(kc), np_f16(kn), Pi, lloyd_max(d, 3))
    vh = Q.decode(np_u32(vc), np_f16(vn), Pi, lloyd_max(d, 1), np_u32(vs), np_f16(vg), S)
    want = OA.softmax_attend(q_np[0].astype(np.float64), kh, vh, 1.0 / math.sqrt(d))
    assert normwise_rel(out.cpu().numpy()[0], want).max() <= 1e-3
