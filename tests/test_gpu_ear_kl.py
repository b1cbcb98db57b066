"""GPU parity: slq_ear_kl against the oracle's binary64 EAR/KL, within 1e-5
absolute per token and for the means."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import Guarded, to_dev_u16, to_host_u16

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _gpu(a_bits, b_bits, tau):
    T = a_bits.shape[0]
    ear = Guarded((T,), torch.float32)
    kl = Guarded((T,), torch.float32)
    means = Guarded((2,), torch.float64)
    A, Bq = to_dev_u16(a_bits), to_dev_u16(b_bits)  # keep both alive during the call
    rc = slq.lib().slq_ear_kl(
        A.data_ptr(), Bq.data_ptr(), T, a_bits.shape[1],
        float(tau), ear.t.data_ptr(), kl.t.data_ptr(), means.t.data_ptr(),
        means.t.data_ptr() + 8, None, torch.cuda.current_stream().cuda_stream)
    assert rc == slq.SLQ_OK
    torch.cuda.synchronize()
    assert ear.intact() and kl.intact() and means.intact()
    m = means.t.cpu().numpy()
    return ear.t.cpu().numpy(), kl.t.cpu().numpy(), m[0], m[1]


@pytest.mark.parametrize("tau", [1.0, 0.7])
@pytest.mark.parametrize("T,V", [(1, 1), (3, 2), (5, 7), (4, 8), (7, 1000), (3, 3001),
                                 (2, 65536 + 24), (3, 151936), (2, 151935)])
def test_matches_oracle(T, V, tau):
    a, b = synth.logits(T, V, seed=T * 31 + V)
    e, k, em, km = _gpu(a, b, tau)
    er, kr = oracle.ear_kl(a, b, tau)
    assert np.abs(e - er).max() <= TOL
    assert np.abs(k - kr).max() <= TOL
    assert abs(em - er.mean()) <= TOL and abs(km - kr.mean()) <= TOL


def test_invariants_on_gpu():
    a, _ = synth.logits(4, 5000, seed=1)
    e, k, _, _ = _gpu(a, a, 1.0)
    assert np.abs(e - 1).max() <= TOL and np.abs(k).max() <= TOL
    la = np.full((2, 64), -1e4)
    lb = np.full((2, 64), -1e4)
    la[:, :32] = 0.0
    lb[:, 32:] = 0.0
    e, _, _, _ = _gpu(synth.to_bf16_bits(la), synth.to_bf16_bits(lb), 1.0)
    assert np.abs(e).max() <= TOL


@pytest.mark.parametrize("tau", [1.0, 0.7])
def test_full_size_sampled_tokens(tau):
    T, V = 4096, 151936
    a, b = synth.logits_torch(T, V)
    ear, kl, em, km = slq.ear_kl(a, b, tau)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(int(tau * 10)).choice(T, size=24, replace=False))
    rows = np.concatenate([[0, T - 1], rows])
    idx = torch.from_numpy(rows).cuda()
    er, kr = oracle.ear_kl(to_host_u16(a.index_select(0, idx)), to_host_u16(b.index_select(0, idx)), tau)
    assert np.abs(ear.index_select(0, idx).cpu().numpy() - er).max() <= TOL
    assert np.abs(kl.index_select(0, idx).cpu().numpy() - kr).max() <= TOL
    # the means are plain averages of the per-token values
    assert abs(em.item() - ear.double().mean().item()) <= 1e-9
    assert abs(km.item() - kl.double().mean().item()) <= 1e-9


def _gpu_topk(a_bits, b_bits, k, tau):
    T = a_bits.shape[0]
    ear = Guarded((T,), torch.float32)
    kl = Guarded((T,), torch.float32)
    means = Guarded((2,), torch.float64)
    A, Bq = to_dev_u16(a_bits), to_dev_u16(b_bits)
    rc = slq.lib().slq_ear_kl_topk(
        A.data_ptr(), Bq.data_ptr(), T, a_bits.shape[1], int(k), float(tau), ear.t.data_ptr(),
        kl.t.data_ptr(), means.t.data_ptr(), means.t.data_ptr() + 8, None,
        torch.cuda.current_stream().cuda_stream)
    assert rc == slq.SLQ_OK
    torch.cuda.synchronize()
    assert ear.intact() and kl.intact() and means.intact()
    m = means.t.cpu().numpy()
    return ear.t.cpu().numpy(), kl.t.cpu().numpy(), m[0], m[1]


@pytest.mark.parametrize("tau", [1.0, 0.7])
@pytest.mark.parametrize("k", [1, 3, 10, 16])
@pytest.mark.parametrize("T,V", [(1, 16), (3, 37), (5, 1000), (4, 4096 + 8), (3, 151936), (2, 151935)])
def test_topk_matches_oracle(T, V, k, tau):
    a, b = synth.logits(T, V, seed=T * 13 + V + k)
    e, kl, em, km = _gpu_topk(a, b, k, tau)
    er, kr, _ = oracle.ear_kl_topk(a, b, k, tau)
    assert np.abs(e - er).max() <= TOL
    assert np.abs(kl - kr).max() <= TOL
    assert abs(em - er.mean()) <= TOL and abs(km - kr.mean()) <= TOL


def test_topk_ties_and_full_k():
    # Ties across threads and units: many equal top logits; the set is the
    # lowest indices among them.
    T, V = 3, 4096
    x = np.full((T, V), -2.0)
    x[:, ::97] = 5.0  # 43 tied maxima, spread over many threads
    x[1, 3000] = 6.0
    a = synth.to_bf16_bits(x)
    b = synth.to_bf16_bits(x + 0.25 * np.sin(np.arange(V)))
    for k in (1, 5, 16):
        e, kl, _, _ = _gpu_topk(a, b, k, 1.0)
        er, kr, _ = oracle.ear_kl_topk(a, b, k, 1.0)
        assert np.abs(e - er).max() <= TOL and np.abs(kl - kr).max() <= TOL
    # K = V on a tiny vocabulary equals the full-vocabulary call.
    a2, b2 = synth.logits(4, 12, seed=5)
    e, kl, _, _ = _gpu_topk(a2, b2, 12, 1.0)
    ef, kf, _, _ = _gpu(a2, b2, 1.0)
    assert np.abs(e - ef).max() <= TOL and np.abs(kl - kf).max() <= TOL


@pytest.mark.parametrize("tau", [1.0, 0.7])
def test_topk_full_size_sampled_tokens(tau):
    T, V = 4096, 151936
    a, b = synth.logits_torch(T, V)
    ear, kl, em, km = slq.ear_kl(a, b, tau, top_k=10)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(int(tau * 10) + 1).choice(T, size=24, replace=False))
    rows = np.concatenate([[0, T - 1], rows])
    idx = torch.from_numpy(rows).cuda()
    er, kr, _ = oracle.ear_kl_topk(to_host_u16(a.index_select(0, idx)), to_host_u16(b.index_select(0, idx)), 10, tau)
    assert np.abs(ear.index_select(0, idx).cpu().numpy() - er).max() <= TOL
    assert np.abs(kl.index_select(0, idx).cpu().numpy() - kr).max() <= TOL
    assert abs(em.item() - ear.double().mean().item()) <= 1e-9
