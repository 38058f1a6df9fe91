"""The staged kernels' bounded waits, run out on purpose without a fault: a
test-only copy of the library is compiled with the consumers' wait limit at
0 ns, so that their wait for a stage's data gives up on an ordinary TMA copy
that is still in flight.  The producer keeps the full 1 s limit for the drain
in which it waits for every load it issued, so no copy is left landing in
shared memory after its CTA exits; with no more layers than ring stages it
never waits for a stage the consumers abandoned.  The call must return, set
CMR_DEVICE_WAIT_TIMEOUT in the status word, and leave the context usable: the
normal library then rotates a fresh batch within the bar."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from tests.helpers import BarStats, oracle_rotate_threads
from vlm_decoder_positional_b200 import build as libbuild
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
WAIT0_LIB = os.path.join(HERE, "_build", "libcmr_wait0.so")


def wait0_library():
    """libcmr built from the package's sources with the consumers' wait limit at 0."""
    srcs = libbuild.sources()
    deps = srcs + [os.path.join(libbuild.CSRC, f) for f in os.listdir(libbuild.CSRC)
                   if f.endswith(".cuh")]
    if not os.path.exists(WAIT0_LIB) or any(os.path.getmtime(p) > os.path.getmtime(WAIT0_LIB)
                                            for p in deps):
        os.makedirs(os.path.dirname(WAIT0_LIB), exist_ok=True)
        tmp = WAIT0_LIB + ".tmp.%d" % os.getpid()
        subprocess.run([libbuild.NVCC] + libbuild.NVCC_FLAGS +
                       ["-DCMR_CONSUMER_WAIT_LIMIT_NS=0", "-I", libbuild.INCLUDE, "-o", tmp] +
                       srcs, check=True)
        os.replace(tmp, WAIT0_LIB)
    lib = ctypes.CDLL(WAIT0_LIB)
    for name in ("cmr_rotate_qk", "cmr_rotate_qk_cache"):
        f = getattr(lib, name)
        f.restype, f.argtypes = cmr.SIGNATURES[name]
    lib.cmr_last_rotate_kernel.restype = ctypes.c_char_p
    return lib


@pytest.mark.parametrize("layers", [1, 2, 3])
def test_consumer_wait_time_out_is_reported_and_the_context_stays_usable(cuda_device, layers):
    dev = cuda_device
    lib = wait0_library()
    n = 8192  # 1,024 tiles: the staged kernel; layers <= 3 ring stages
    assert cmr.rotate_qk_kernel(n, layers, 8, 2) == "rotate_qk_staged_kernel"
    q = inputs.random_qk((layers, n, 8, 256), 1, dev)
    k = inputs.random_qk((layers, n, 2, 256), 2, dev)
    pos = torch.randint(0, 9000, (3, n), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sec = (ctypes.c_int32 * 3)(11, 11, 10)
    with torch.cuda.device(dev):
        rc = lib.cmr_rotate_qk(q.data_ptr(), k.data_ptr(), pos.data_ptr(), n, layers, 8, 2, 256,
                               1e7, sec, 64, status.data_ptr(),
                               torch.cuda.current_stream(dev).cuda_stream)
    assert rc == cmr.CMR_OK
    assert lib.cmr_last_rotate_kernel() == b"rotate_qk_staged_kernel"
    torch.cuda.synchronize()  # the kernel returned; no error is pending
    assert int(status.item()) & cmr.CMR_DEVICE_WAIT_TIMEOUT

    # the same context, the normal library, a fresh batch
    q2 = inputs.random_qk((layers, n, 8, 256), 3, dev)
    k2 = inputs.random_qk((layers, n, 2, 256), 4, dev)
    q_in = q2.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    k_in = k2.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    status2 = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.rotate_qk(q2, k2, pos, device_status=status2)
    torch.cuda.synchronize()
    assert int(status2.item()) == 0
    p = pos.cpu().numpy()
    BarStats("q after a time-out").add(q2.cpu().view(torch.int16).numpy().view(np.uint16),
                                       oracle_rotate_threads(q_in, p)).check()
    BarStats("k after a time-out").add(k2.cpu().view(torch.int16).numpy().view(np.uint16),
                                       oracle_rotate_threads(k_in, p)).check()


def test_cache_form_consumer_wait_time_out_is_reported(cuda_device):
    dev = cuda_device
    lib = wait0_library()
    n, layers = 8192, 2
    assert cmr.rotate_qk_cache_kernel(n, layers, 8, 2) == "rotate_qk_cache_staged_kernel"
    cu = torch.tensor([0, n], dtype=torch.int32, device=dev)
    start = torch.tensor([1 << 30], dtype=torch.int32, device=dev)
    amount = torch.zeros(1, dtype=torch.int32, device=dev)
    q = inputs.random_qk((layers, n, 8, 256), 5, dev)
    k = inputs.random_qk((layers, n, 2, 256), 6, dev)
    v = inputs.random_qk((layers, n, 2, 256), 7, dev)
    kc = torch.zeros((layers, 1, 2, n, 256), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sec = (ctypes.c_int32 * 3)(11, 11, 10)
    with torch.cuda.device(dev):
        # the first launch of this form in the process sets its shared-memory
        # opt-in (outside any capture)
        rc = lib.cmr_rotate_qk_cache(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu.data_ptr(), 1,
                                     None, start.data_ptr(), amount.data_ptr(), n, layers, 8, 2,
                                     256, 1e7, sec, 64, kc.data_ptr(), vc.data_ptr(), 1, n, None,
                                     status.data_ptr(), torch.cuda.current_stream(dev).cuda_stream)
    assert rc == cmr.CMR_OK
    assert lib.cmr_last_rotate_kernel() == b"rotate_qk_cache_staged_kernel"
    torch.cuda.synchronize()
    assert int(status.item()) & cmr.CMR_DEVICE_WAIT_TIMEOUT
