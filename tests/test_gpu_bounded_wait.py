"""Failure detection on the device: a bounded wait that nothing completes gives up,
records the timeout in the device error word and lets its kernel return; the host
reads HLA_ERR_TIMEOUT from hla_device_status, clears it, and the context keeps
working (a prefill still matches the oracle afterwards).  Nothing faults, traps or
hangs: the wait is limited to 2 ms."""
import numpy as np
import pytest
import torch

import hla_synth as syn
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hla():
    import gated_delta_rule_transitions_b200 as m
    m.lib()
    return m._hla


def test_completed_wait_reports_nothing(hla):
    hla.hla_device_status(clear=True)
    hla.hla_check_bounded_wait(2000, complete=True)
    st, code = hla.hla_device_status(clear=True)
    assert st == hla.HLA_OK and code == 0


def test_expired_wait_is_reported_and_context_stays_usable(hla):
    hla.hla_device_status(clear=True)
    hla.hla_check_bounded_wait(2000, complete=False)
    st, code = hla.hla_device_status(clear=False)
    assert st == hla.HLA_ERR_TIMEOUT and (code & 1) == 1
    assert "bounded device wait" in hla.last_error()
    st, code = hla.hla_device_status(clear=True)   # read and clear
    assert st == hla.HLA_ERR_TIMEOUT
    st, code = hla.hla_device_status(clear=True)
    assert st == hla.HLA_OK and code == 0
    # the context is intact: a small prefill still matches the oracle
    w = syn.TINY_F32
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    for h in range(w.H):
        r = P.oracle_prefill_head(w, inp, 0, h)
        P.check_f32(P.np64(o[0, :, h]), r.o)
    st, code = hla.hla_device_status(clear=True)
    assert st == hla.HLA_OK
