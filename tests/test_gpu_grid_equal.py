"""GPU parity for mx_grid_equal, and the fault-injection protocol of "End-to-End MXFP8
Reinforcement Learning on Blackwell" (Table 13) as far as a byte comparison can see it:
each injected violation is made in host memory and the device comparison must report the exact
number of differing bytes and the first index; an untouched copy must report (0, -1)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import scale_positions, to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def gpu_compare(a_np: np.ndarray, b_np: np.ndarray, offset: int = 0):
    """Copies a and b to the device (optionally at a byte offset, to exercise unaligned buffers) and
    runs mx_grid_equal through the C ABI."""
    n = a_np.size
    da = torch.zeros(n + 32, dtype=torch.uint8, device="cuda")
    db = torch.zeros(n + 32, dtype=torch.uint8, device="cuda")
    da[offset: offset + n] = torch.from_numpy(a_np)
    db[offset: offset + n] = torch.from_numpy(b_np)
    cnt, first = mx.grid_equal(da[offset: offset + n], db[offset: offset + n])
    return int(cnt.item()), int(first.item())


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 4096, 100003, 1 << 22])
@pytest.mark.parametrize("offset", [0, 3])
def test_random_buffers_match_oracle(n, offset):
    a = synth.random_bytes(n, seed=n).numpy()
    b = a.copy()
    g = np.random.default_rng(n + offset)
    for k in (0, 1, 5):
        if n == 0:
            break
        idx = g.choice(n, min(k, n), replace=False)
        b[idx] ^= np.uint8(0x5A)
        assert gpu_compare(a, b, offset) == oracle.grid_equal(a, b)


def test_grid_equal_multi_matches_oracle():
    # 700 pairs (more than one launch holds): mixed sizes, zero-length, unaligned views, faults.
    g = np.random.default_rng(11)
    host, pairs = [], []
    pool_a = torch.zeros(48 << 20, dtype=torch.uint8, device="cuda")
    pool_b = torch.zeros(48 << 20, dtype=torch.uint8, device="cuda")
    off = 0
    for i in range(700):
        n = int(g.choice([0, 1, 15, 16, 100, 4096, 32768, 40000, 70001]))
        a = synth.random_bytes(n, seed=i).numpy()
        b = a.copy()
        if n and g.random() < 0.5:
            idx = g.choice(n, min(n, int(g.integers(1, 4))), replace=False)
            b[idx] ^= np.uint8(0x81)
        shift = int(g.integers(0, 3))         # some views start off 16-byte alignment
        if off + shift + n > pool_a.numel():
            break
        pool_a[off + shift: off + shift + n] = torch.from_numpy(a)
        pool_b[off + shift: off + shift + n] = torch.from_numpy(b)
        pairs.append((pool_a[off + shift: off + shift + n], pool_b[off + shift: off + shift + n]))
        host.append((a, b))
        off += shift + n + 16 - (shift + n) % 16
    cnt, first = mx.grid_equal_multi(pairs)
    cnt, first = to_np(cnt), to_np(first)
    for i, (a, b) in enumerate(host):
        assert (int(cnt[i]), int(first[i])) == oracle.grid_equal(a, b), i
    assert len(host) > 512


def test_large_buffer_single_fault_at_the_end():
    # "corruption confined to ... a late layer": one byte in the last 16 bytes of 1 GiB.
    n = 1 << 30
    a = torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda")
    b = a.clone()
    b[n - 5] ^= 1
    cnt, first = mx.grid_equal(a, b)
    assert (int(cnt.item()), int(first.item())) == (1, n - 5)
    cnt, first = mx.grid_equal(a, a.clone())
    assert (int(cnt.item()), int(first.item())) == (0, -1)


class TestFaultInjection:
    """Learner grid from the oracle; sampler copy = that grid with one Table 13 violation."""

    @pytest.fixture(scope="class")
    def grid(self):
        W = synth.sync_weight(3, 0, rows=512, cols=1024)
        q, s = oracle.quantize_rowwise(W)
        return W, q, s, oracle.swizzle(s)

    def test_untouched_copy(self, grid):
        _, q, s, sw = grid
        for x in (q, s, sw):
            assert gpu_compare(x.reshape(-1), x.reshape(-1).copy()) == (0, -1)

    def test_one_flipped_data_byte(self, grid):
        _, q, _, _ = grid
        b = q.copy()
        b[300, 77] ^= 0x01
        assert gpu_compare(q.reshape(-1), b.reshape(-1)) == (1, 300 * 1024 + 77)

    def test_new_weights_with_stale_scales(self, grid):
        # The sampler took the new data but kept the previous step's raw and swizzled scales.
        W, q, s, sw = grid
        W2 = (W.float() * 2.0).to(torch.bfloat16)             # every scale moves by one
        q2, s2 = oracle.quantize_rowwise(W2)
        assert gpu_compare(q.reshape(-1), q2.reshape(-1)) == oracle.grid_equal(q, q2)
        n, first = gpu_compare(s2.reshape(-1), s.reshape(-1))
        assert n == s.size and first == 0
        n, first = gpu_compare(oracle.swizzle(s2), sw)
        assert n == s.size and first == 0                      # pads agree, every scale differs

    def test_stale_swizzled_copy_only(self, grid):
        # F3: raw scales fresh, the derived interleaved copy stale in one 128-row block.
        _, q, s, sw = grid
        stale = sw.copy()
        pos = scale_positions(*s.shape)
        rows = np.arange(128, 256)
        stale[pos[rows].reshape(-1)] ^= 0x10
        assert gpu_compare(s.reshape(-1), s.reshape(-1).copy()) == (0, -1)
        n, first = gpu_compare(sw, stale)
        assert n == 128 * s.shape[1] and first == int(pos[rows].min())

    def test_permuted_rows_same_shape_and_dtype(self, grid):
        # F4: an in-place repack that keeps shape and dtype (rows of one block permuted).
        _, q, _, _ = grid
        perm = q.copy()
        perm[64:96] = q[64:96][::-1]
        exp = oracle.grid_equal(q, perm)
        assert exp[0] > 0 and gpu_compare(q.reshape(-1), perm.reshape(-1)) == exp

    def test_corruption_in_last_tensor_of_many(self):
        # 144 tensors (36 layers x 4), corruption only in the last one.
        tensors = [synth.random_bytes(4096 + 16 * i, seed=i).numpy() for i in range(144)]
        for i, t in enumerate(tensors):
            b = t.copy()
            if i == 143:
                b[-1] ^= 0xFF
            res = gpu_compare(t, b)
            assert res == ((1, t.size - 1) if i == 143 else (0, -1))


def test_bounded_wait_expires_and_context_stays_usable():
    mx.device_error()
    mx.set_wait_timeout_ns(20_000_000)          # 20 ms
    try:
        st = mx.lib().mx_diag_expired_wait(None)
        assert st == 0
        assert mx.device_error() == 1
    finally:
        mx.set_wait_timeout_ns(0)
    # The context still works after the expired wait.
    a = torch.arange(1000, dtype=torch.int32, device="cuda").to(torch.uint8)
    cnt, first = mx.grid_equal(a, a.clone())
    assert int(cnt.item()) == 0 and int(first.item()) == -1
    assert mx.device_error() == 0
