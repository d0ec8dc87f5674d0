"""Failure detection on the GPU without a GPU fault: a bounded device-side wait
that can never complete gives up after its limit, reports the timeout through
the status word, makes later waits of the aborting CTA return at once, and
leaves the CUDA context usable for the next launch."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_attention_38_b200 as pkv
from paged_kv_attention_38_b200 import workloads as W

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT = 1  # the status code a timed-out wait records


def test_bounded_wait_times_out_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    times = torch.zeros(2, dtype=torch.int64, device="cuda")
    assert pkv.load_library().pkv_selftest_wait_timeout(status.data_ptr(), times.data_ptr(), None) == pkv.PKV_OK
    torch.cuda.synchronize()
    assert int(status.item()) == WAIT_TIMEOUT
    first, second = (int(x) for x in times.cpu())
    assert 1.9e9 <= first < 10e9, first      # gave up after the 2 s limit, not before, not much after
    assert 0 <= second < 1e6, second         # the aborting CTA's next wait returned at once
    # the context is still usable: a small prefill still matches the oracle
    p = W.tiny_prefill()
    idx = torch.from_numpy(p.kv_indices.astype(np.int32)).cuda()
    pl = pkv.plan(p.qo_indptr, p.kv_indptr, idx, p.kv_last_page_len, p.num_qo_heads, p.num_kv_heads, p.head_dim,
                  p.page_size, p.causal, p.sm_scale)
    o, lse = pkv.run(pl, p.q.cuda(), p.k_cache.cuda(), p.v_cache.cuda())
    torch.cuda.synchronize()
    assert pkv.device_status(pl) == 0
    o_ref, l_ref = oracle.paged_attention(p.q, p.k_cache, p.v_cache, p.qo_indptr, p.kv_indptr, p.kv_indices,
                                          p.kv_last_page_len, p.page_size, p.causal, p.sm_scale)
    o_g = o.float().cpu().double().numpy()
    assert np.all(np.abs(o_g - o_ref) <= 1e-2 + 1e-2 * np.abs(o_ref))
    assert np.all(np.abs(lse.cpu().double().numpy() - l_ref) <= 1e-3)
