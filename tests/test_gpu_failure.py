"""Failure path on the GPU without a fault: a kernel's bounded mbarrier wait
runs out (nothing arrives on its barrier), the host reads MSA_ERR_TIMEOUT
from msa_sync_check, and the context stays usable for the next call."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import DevBank, host_normal, route_gpu

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    import routed_sparse_attention_msa_b200 as msa
    msa.sync_check()  # nothing pending before the probe
    msa.wait_probe()
    with pytest.raises(msa.MsaError) as err:
        msa.sync_check()
    assert err.value.code == 5  # MSA_ERR_TIMEOUT
    msa.sync_check()  # the flag was taken: the next check is clean
    # the context still routes correctly
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 0, content=False)
    qr = host_normal((4, 8, 128), synth.tid("q_noise", 0, 5))
    qso = np.array([0, 4], np.int32)
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    np.testing.assert_allclose(alls, o_all, atol=1e-3, rtol=0)
