"""A bounded wait that runs out ends the kernel with a status, not a hang.

Every wait of the decode kernels on a shared-memory copy gives up after a
time limit, records BASISKV_STATUS_TIMEOUT and drains the copies it did
issue before returning.  The test build of the library (BASISKV_WAIT_TEST:
1 ms limit, and the first warp of each grid, or in the shared-ring
attention kernel the first CTA, never issues the copies of its second item)
makes such a wait run out on purpose: nothing faults, no copy
is left in flight, the call returns, the status says TIMEOUT, and the CUDA
context stays usable, so a following call of the normal library on a fresh
handle is correct.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import workloads as W
from oracle import oracle
from helpers import to_problem
from test_gpu_parity import OUT_TOL, out_error, gpu_decode

pytestmark = pytest.mark.gpu


# k = 16 pages (32 stages per unit) runs the per-warp-ring attention kernel,
# k = 48 (96 stages) the shared-ring one
@pytest.mark.parametrize("topk", [16, 48])
def test_wait_runs_out_and_is_reported(topk):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    from compressed_kv_cache_routing_b200 import build
    build.build()
    lib = bk.load(build.build_wait_test())
    spec = W.shrink("llama3_8b_decode", batch=3, len_lo=4096, len_hi=4096, topk=topk)
    w = W.generate(spec, device="cuda")
    s = w.spec
    ref = bk.BasisKV.for_workload(w)            # normal library: only for its params
    p = bk.basiskv_params.from_buffer_copy(ref.params)
    h = ctypes.c_void_p()
    assert lib.basiskv_create(ctypes.byref(p), ctypes.byref(h)) == 0, lib.basiskv_last_error()
    pt = np.ascontiguousarray(np.where(w.page_table >= 0, w.page_table, 0), np.int32)
    lens = np.ascontiguousarray(w.seq_lens, np.int32)
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.basiskv_load_page_table(h, s.batch, pt.ctypes.data, pt.shape[1], lens.ctypes.data, stream) == 0
    out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
    sel = torch.full((s.batch, s.num_kv_heads, s.topk), -7, device="cuda", dtype=torch.int32)
    t0 = time.perf_counter()
    rc = lib.basiskv_decode_attn(h, s.batch, w.q.data_ptr(), s.topk, s.softmax_scale, out.data_ptr(),
                                 sel.data_ptr(), stream)
    assert rc == 0, lib.basiskv_last_error()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    st = ctypes.c_uint32()
    assert lib.basiskv_get_status(h, ctypes.byref(st), 1) == 0
    assert st.value & bk.BASISKV_STATUS_TIMEOUT, st.value
    assert elapsed < 5.0, elapsed
    launch = (ctypes.c_int * 6)()
    assert lib.basiskv_last_launch(h, ctypes.byref(launch)) == 0
    assert launch[4] == 1 and launch[5] == (2 if topk == 48 else 1)  # the persistent tensor-core kernels ran
    assert lib.basiskv_get_status(h, ctypes.byref(st), 0) == 0 and st.value == 0  # cleared
    assert lib.basiskv_destroy(h) == 0
    ref.close()
    # the context is intact: the normal library on a fresh handle is right
    ref_out, ref_sel, _, _ = oracle.decode(to_problem(w))
    o, sl = gpu_decode(w)
    assert np.array_equal(sl, ref_sel)
    assert out_error(o, ref_out) <= OUT_TOL
