"""The device error path: a kernel that meets an inconsistent input skips
the access and records a code in the library's device error word, and the
host reads it as LSA_EDEVICE from lsa_check_device_error() (which also
clears it).  The failure is made on the host, by an index entry past the
end of K; no access leaves the buffers."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import clustered_key_indexing_b200 as m
    return m


def test_index_past_end_raises_edevice(lsa):
    from clustered_key_indexing_b200._lib import LSA_EDEVICE, LSAError
    rng = np.random.default_rng(11)
    T, hq, hkv, nq, n = 96, 8, 2, 5, 40
    Q = oracle.bf16_rne(rng.standard_normal((nq, hq, 128))).reshape(nq, hq, 128)
    K = oracle.bf16_rne(rng.standard_normal((T, hkv, 128))).reshape(T, hkv, 128)
    V = oracle.bf16_rne(rng.standard_normal((T, hkv, 128))).reshape(T, hkv, 128)
    idx = np.stack([rng.permutation(T)[:n] for _ in range(nq * hkv)]).astype(np.int32).reshape(nq, hkv, n)
    bad = idx.copy()
    bad[2, 1, 7] = T          # one entry past the end of K
    lsa.check_device_error()  # start from a clear word
    O = lsa.sparse_attn(to_dev_bf16(Q), to_dev_bf16(K), to_dev_bf16(V), to_dev(bad), T=T)
    torch.cuda.synchronize()
    with pytest.raises(LSAError) as ei:
        lsa.check_device_error()
    assert ei.value.status == LSA_EDEVICE
    assert "index entry" in str(ei.value)
    lsa.check_device_error()  # reading the word cleared it
    # the entry was skipped: the output equals attention over the list without it
    skip = bad.copy()
    skip[2, 1, 7] = -1
    ref = oracle.attention(Q, K, V, skip)
    e = np.abs(O.float().cpu().numpy().astype(np.float64) - ref)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3
