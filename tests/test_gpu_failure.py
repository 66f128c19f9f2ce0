"""Failure detection on the GPU without a fault: a bounded wait of the
tensor-core indexer is made to run out (a barrier that nothing completes,
with every wait of the launch limited to 2 ms).  The kernel returns on its
own, the workspace's status word reports V4A_ERR_TIMEOUT, the context stays
usable, and the next normal call on the same workspace is correct."""
import numpy as np
import pytest
import torch

import synth
from oracle import indexer as oidx
from tests.gpu_util import check_topk, code_rows, desc_for, dev, read_keys, v4

pytestmark = pytest.mark.gpu

ST_TIMEOUT = 1 << 8


def test_bounded_wait_runs_out_and_the_next_call_succeeds():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    v = v4()
    rng = np.random.default_rng(17)
    B, N, H_I, d_I, k = 2, 4096, 64, 128, 256
    ly = synth.Layer("csa", 4, 64, 512, 64, 128, H_I, d_I, k)
    desc = desc_for(ly)
    keys = rng.standard_normal((B, N, d_I)).astype(np.float32)
    qI = rng.standard_normal((B, H_I, d_I)).astype(np.float32)
    w = rng.uniform(0, 1, (B, H_I)).astype(np.float32)
    positions = np.array([4 * N - 1, 4 * 3000 + 1])
    krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
    qrows, qsf = code_rows(desc, dev(qI.reshape(1, B * H_I, d_I)), v.MXFP4)
    qrows, qsf = qrows.reshape(B, H_I, -1), qsf.reshape(B, H_I, -1)
    kw = dict(qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64), keys=krows,
              keys_sf=ksf, key_rows=N, max_vis=N, B=B)
    ws = v.workspace(desc, B, N)
    scores = torch.zeros(B, N, dtype=torch.float32, device="cuda")
    v.debug_index_stall(desc, ws=ws, wait_ns=2_000_000, scores_out=scores, **kw)
    st, bits = v.device_status_code(ws)
    assert st == 5, (st, hex(bits))                     # V4A_ERR_TIMEOUT
    assert bits & ST_TIMEOUT
    # the context is intact: a plain torch op and a normal call on the same workspace
    assert float(torch.ones(4, device="cuda").sum()) == 4.0
    v.workspace_init(ws)
    idx = torch.full((B, k), -3, dtype=torch.int32, device="cuda")
    v.index_topk(desc, ws=ws, idx_out=idx, scores_out=scores, **kw)
    assert v.device_status(ws) == 0
    kd, qd = read_keys(krows, ksf, v.MXFP4), read_keys(qrows, qsf, v.MXFP4)
    g_s, g_i = scores.cpu().numpy(), idx.cpu().numpy()
    for b in range(B):
        nv = (int(positions[b]) + 1) // 4
        s = oidx.scores(qd[b], w[b], kd[b, :nv])
        assert np.max(np.abs(g_s[b, :nv] - s)) <= 1e-5 * max(1.0, np.max(np.abs(s)))
        check_topk(g_i[b], s, nv, k)
