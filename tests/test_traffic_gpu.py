"""The memory-floor replay (msda_debug_row_traffic) does exactly the row
traffic it claims: every listed row is gathered once (mode 0, checked
through the sums it leaves in the sink), reduced once (mode 1: grad counts
the rows' occurrences) or gathered and reduced (mode 2), and rows outside
the buffers or off the vector grid (4 elements for fp32 value, 8 for bf16)
are skipped."""
import numpy as np
import pytest
import torch

from scale_deformable_attention_02_b200 import msda_debug_row_traffic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rows(n_rows_map, count, seed):
    rng = np.random.default_rng(seed)
    r = rng.integers(0, n_rows_map, count) * 32  # element offsets of 128-byte rows
    r[:7] = [-32, n_rows_map * 32, 5, 0, 0, 32, n_rows_map * 32 - 32]  # 3 skipped, repeats
    return r.astype(np.int32)


def test_row_traffic_modes():
    n_map = 5000
    value = torch.randn(n_map * 32, device="cuda")
    rows = _rows(n_map, 200_003, 1)
    valid = (rows >= 0) & (rows + 32 <= n_map * 32) & (rows % 4 == 0)
    vr = value.cpu().numpy().reshape(-1)
    trows = torch.from_numpy(rows).cuda()
    ctas = 16
    sink = torch.zeros(ctas * 256, device="cuda")
    msda_debug_row_traffic(0, trows, value=value, sink=sink, ctas=ctas)
    expect = sum(vr[o:o + 32].astype(np.float64).sum() for o in rows[valid])
    assert abs(float(sink.double().sum()) - expect) <= 1e-3 * (1 + abs(expect))
    grad = torch.zeros_like(value)
    msda_debug_row_traffic(1, trows, grad=grad, ctas=ctas)
    counts = np.bincount(rows[valid] // 32, minlength=n_map).astype(np.float32)
    np.testing.assert_array_equal(grad.cpu().numpy().reshape(n_map, 32),
                                  np.repeat(counts[:, None], 32, axis=1))
    grad.zero_()
    msda_debug_row_traffic(2, trows, value=value, grad=grad)
    np.testing.assert_allclose(grad.cpu().numpy().reshape(n_map, 32),
                               counts[:, None] * vr.reshape(n_map, 32), rtol=1e-5, atol=1e-4)


def test_row_traffic_bf16_value():
    """bf16 value rows (64 bytes) gathered, and added into an fp32 gradient
    (128-byte rows); offsets must sit on the 8-element grid."""
    n_map = 3000
    value = torch.randn(n_map * 32, device="cuda").to(torch.bfloat16)
    rows = _rows(n_map, 100_001, 2)
    rows[7:9] = [4, 36]  # on the fp32 grid, off the bf16 one: skipped
    valid = (rows >= 0) & (rows + 32 <= n_map * 32) & (rows % 8 == 0)
    vr = value.float().cpu().numpy().reshape(-1)
    trows = torch.from_numpy(rows).cuda()
    ctas = 16
    sink = torch.zeros(ctas * 256, device="cuda")
    msda_debug_row_traffic(0, trows, value=value, sink=sink, ctas=ctas, depth=4)
    expect = sum(vr[o:o + 32].astype(np.float64).sum() for o in rows[valid])
    assert abs(float(sink.double().sum()) - expect) <= 1e-3 * (1 + abs(expect))
    grad = torch.zeros(n_map * 32, device="cuda")
    msda_debug_row_traffic(2, trows, value=value, grad=grad, ctas=ctas)
    counts = np.bincount(rows[valid] // 32, minlength=n_map).astype(np.float32)
    np.testing.assert_allclose(grad.cpu().numpy().reshape(n_map, 32),
                               counts[:, None] * vr.reshape(n_map, 32), rtol=1e-5, atol=1e-4)
