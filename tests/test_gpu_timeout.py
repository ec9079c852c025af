"""The bounded-wait path: a device wait that runs out reports DSA_ERR_TIMEOUT and the
kernel returns, leaving the context usable.

No fault is provoked.  The host sets the workspace's test word (DSA_TEST_WITHHOLD_TILE);
the indexer's TMA producer then never sends its first key tile, so the MMA issuer's and
the epilogue's waits on it give up after their limit (about 2 s), record the timeout in
the status word, release their tensor memory and exit.  A normal call on the same device
afterwards must still be correct.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
WITHHOLD = 0x5D5A7E57


def _hooked_call(B, n_q, q_pos0, n_kv, H, d, topk):
    q, k, w = synth.integer_indexer("timeout", B, n_kv, H, d, -3, 3, q_rows=n_q)
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H, d, topk), dtype=torch.uint8,
                     device=DEV)
    ws.view(torch.int32)[2] = WITHHOLD
    dsa.idx_score_topk(q.to(DEV), k.to(DEV), w.to(DEV), topk, q_pos0=q_pos0, workspace=ws)
    with pytest.raises(dsa.DsaError) as err:
        dsa.check_status(ws)
    assert err.value.code == dsa.DSA_ERR_TIMEOUT
    assert "timed out" in str(err.value)
    # the status word was cleared by the check; clear the hook and run the same call normally
    ws.view(torch.int32)[2] = 0
    idx = dsa.idx_score_topk(q.to(DEV), k.to(DEV), w.to(DEV), topk, q_pos0=q_pos0, workspace=ws)
    assert dsa.read_status(ws) == 0
    idx = idx.cpu().numpy()
    for b in range(B):
        sc = oracle.indexer_scores(q[b], k[b], w[b], q_pos0)
        assert np.array_equal(idx[b], oracle.topk_select(sc, topk, q_pos0))


def test_prefill_indexer_wait_times_out_and_recovers():
    # one work tile, one key tile: a single CTA whose only key tile is withheld
    _hooked_call(1, 16, 0, 128, 32, 128, 8)


def test_decode_indexer_wait_times_out_and_recovers():
    # one query against 1024 keys: the split decode kernel (8 key tiles, one unit)
    _hooked_call(1, 1, 1023, 1024, 32, 128, 64)
