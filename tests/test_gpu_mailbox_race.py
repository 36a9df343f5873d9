"""The mailbox slot protocol with producers and consumer running at the same time.

The other mailbox tests finish every producer of a round before its consumer
starts. Here one cooperative launch (tests/csrc/mailbox_race.cu) plays a whole
round on one GPU: W producer blocks store their rows with the library's
producer step after per-row delays of up to tens of microseconds, while the
consumer blocks read the same slots with the library's bounded slot wait, sum
them in producer order and re-mark them. All blocks are resident at once (a
cooperative launch), so the consumer's waits run while the stores are in
flight; no kernel waits on another launch.

* The consumer's sums are bitwise the fp32 sums of the producers' rows taken in
  producer order, a negative zero in a row counting as positive zero.
* The consumer did meet unwritten elements (the count of 8-byte groups whose
  first load still held the mark is positive), so the waits were exercised.
* Every slot element is back to negative zero afterwards, and no error is
  recorded.
* A row that one producer never stores makes the consumer's wait run out (a
  short budget): MHC_ERR_DEVICE_TIMEOUT is recorded, that row's sum leaves the
  producer out, every other row is exact, and the next round on the same
  context goes through.
"""

import ctypes

import numpy as np
import pytest
import torch

from mhc_residual_stream_b200 import build

NEG_ZERO = 0x8000
DEVICE_TIMEOUT = 5  # MHC_ERR_DEVICE_TIMEOUT
WAITS = []  # (case, 8-byte groups the consumer first loaded unwritten, groups read); printed after a GPU run


def _lib():
    L = ctypes.CDLL(build.build_race_check())
    L.mhc_race_run.restype = ctypes.c_int
    L.mhc_race_run.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 4 + [ctypes.c_int64, ctypes.c_void_p]
    L.mhc_race_max_delay_cycles.restype = ctypes.c_int
    return L


def test_race_library_builds_and_exports():
    """Host only: the check's library compiles for sm_100a and exports its entry points."""
    L = _lib()
    assert L.mhc_race_max_delay_cycles() > 0
    assert hasattr(L, "mhc_race_run")
    # argument checks run before any CUDA call
    assert L.mhc_race_run(None, None, None, None, None, 2, 1, 64, 1, 1000, None) == -1


def _rows(W, R, H, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(W, R, H, generator=g).to(torch.bfloat16)
    bits = x.view(torch.int16)
    # exact zeros of both signs, which the producers must store as positive zero
    z = torch.rand(W, R, H, generator=g) < 0.01
    bits[z] = 0
    nz = torch.rand(W, R, H, generator=g) < 0.01
    bits[nz] = -32768  # 0x8000
    return x


def _expected(x: torch.Tensor, skip=None) -> np.ndarray:
    """fp32 sums in producer order; `skip` = (w, r): producer w left out of row r."""
    xf = x.float().numpy()
    W, R, H = xf.shape
    s = np.zeros((R, H), dtype=np.float32)
    for u in range(W):
        add = xf[u].copy()
        if skip is not None and skip[0] == u:
            add[skip[1]] = 0.0
        s = (s + add).astype(np.float32)
    return s


def _run(L, x, delays, consumers, budget_ns):
    W, R, H = x.shape
    dev = torch.device("cuda", 0)
    assert delays.shape == (W, R) and int(delays.max()) <= L.mhc_race_max_delay_cycles()
    xd = x.to(dev)
    slots = torch.full((W, R, H), -32768, dtype=torch.int16, device=dev)  # 0x8000 everywhere
    out = torch.full((R, H), float("nan"), dtype=torch.float32, device=dev)
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    d = torch.as_tensor(delays, dtype=torch.int32).to(dev)
    rc = L.mhc_race_run(xd.data_ptr(), slots.data_ptr(), out.data_ptr(), status.data_ptr(), d.data_ptr(), W, R, H,
                        consumers, budget_ns, torch.cuda.current_stream().cuda_stream)
    assert rc == 0, f"launch failed: {rc}"
    torch.cuda.synchronize()
    return out.cpu().numpy(), status.cpu().numpy().view(np.uint32), slots.cpu().numpy().view(np.uint16)


@pytest.mark.gpu
@pytest.mark.parametrize("W,R,H,max_delay,seed", [
    (2, 4, 7168, 100_000, 1),     # two producers, the decode row width
    (8, 16, 7168, 100_000, 2),    # P = 8 producers, 16 rows
    (16, 2, 7168, 60_000, 3),     # the largest group
    (3, 5, 1032, 40_000, 4),      # a row width that is not a multiple of the consumer's stride
])
def test_concurrent_round_is_exact(W, R, H, max_delay, seed):
    L = _lib()
    x = _rows(W, R, H, seed)
    rng = np.random.default_rng(seed)
    delays = rng.integers(0, max_delay, size=(W, R)).astype(np.int32)
    got, status, slots = _run(L, x, delays, consumers=8, budget_ns=500_000_000)
    WAITS.append((f"W={W} R={R} H={H}", int(status[1]), W * R * H // 4))
    assert status[0] == 0
    assert status[1] > 0, "the consumer never met an unwritten element: nothing ran concurrently"
    want = _expected(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.all(slots == NEG_ZERO)


@pytest.mark.gpu
def test_producers_storing_at_once():
    """No delays: the stores race the consumer's first loads from the start."""
    L = _lib()
    x = _rows(4, 8, 4096, 7)
    got, status, slots = _run(L, x, np.zeros((4, 8), dtype=np.int32), consumers=4, budget_ns=500_000_000)
    assert status[0] == 0
    assert np.array_equal(got.view(np.uint32), _expected(x).view(np.uint32))
    assert np.all(slots == NEG_ZERO)


@pytest.mark.gpu
def test_row_never_stored_runs_out_and_next_round_goes_through():
    L = _lib()
    W, R, H = 4, 3, 1024
    x = _rows(W, R, H, 11)
    delays = np.full((W, R), 20_000, dtype=np.int32)
    delays[2, 1] = -1  # producer 2 never stores row 1
    got, status, slots = _run(L, x, delays, consumers=2, budget_ns=2_000_000)
    assert status[0] == DEVICE_TIMEOUT
    want = _expected(x, skip=(2, 1))
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.all(slots == NEG_ZERO)
    # the context is still usable: a complete round afterwards is exact
    delays[2, 1] = 20_000
    got, status, _ = _run(L, x, delays, consumers=2, budget_ns=500_000_000)
    assert status[0] == 0
    assert np.array_equal(got.view(np.uint32), _expected(x).view(np.uint32))
