"""The debug build (BASISKV_DEBUG) checks the indices the kernels keep in
range by construction and reports a failed check as
BASISKV_STATUS_DEBUG_BOUNDS.  On valid inputs no check fails, and the checks
change no arithmetic: outputs and selections are bit-identical to the normal
build's, for both attention kernels, int8 keys included."""
import ctypes

import numpy as np
import pytest
import torch

from compressed_kv_cache_routing_b200 import basiskv as bk
from compressed_kv_cache_routing_b200 import workloads as W
from test_gpu_parity import SMALL, gpu_decode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["llama3_8b_decode", "llama_shared_ring", "long_context", "high_concurrency"])
def test_debug_build_matches_and_reports_nothing(name):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    from compressed_kv_cache_routing_b200 import build
    build.build()
    lib = bk.load(build.build_debug())
    w = W.generate(SMALL[name], device="cuda")
    s = w.spec
    ref_out, ref_sel = gpu_decode(w)
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
    for _ in range(2):
        assert lib.basiskv_decode_attn(h, s.batch, w.q.data_ptr(), s.topk, s.softmax_scale, out.data_ptr(),
                                       sel.data_ptr(), stream) == 0, lib.basiskv_last_error()
    torch.cuda.synchronize()
    st = ctypes.c_uint32()
    assert lib.basiskv_get_status(h, ctypes.byref(st), 1) == 0
    assert st.value == 0, st.value
    assert np.array_equal(out.cpu().numpy(), ref_out) and np.array_equal(sel.cpu().numpy(), ref_sel)
    assert lib.basiskv_destroy(h) == 0
    ref.close()
