"""Per-axis scaling of the distance on the GPU (the time scale of the review
thread on the FPS arguments, graphnet PR #923): both points' coordinates are
multiplied by the axis weights in float32 before the fixed-order distance.
Every schedule, the Lloyd and kNN paths and the standalone calls are compared
with the CPU oracle under the same weights (indices and labels bit-exact,
floats within the parity tolerance), and unit weights give the same bits as
no weights."""
import numpy as np
import pytest

import oracle
import workloads
from parity import compare, run_gpu, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import farthest_point_sampling_b200 as fps  # noqa: E402

TIME_SCALE = (1.0, 1.0, 1.0, 0.3)      # ns weighted down against metres
MIXED = (0.5, 2.0, 1.0, 0.0625)         # powers of two, time nearly ignored


@pytest.mark.parametrize("schedule,sizes", [(0, [5, 130, 200, 448, 300]), (1, [700, 2560, 129]),
                                            (2, [3000, 12288]), (3, [40000, 13000]), (4, [120000])])
@pytest.mark.parametrize("w", [TIME_SCALE, MIXED])
def test_schedules_match_the_oracle_under_axis_weights(schedule, sizes, w):
    b = workloads.random_batch(700 + schedule, sizes, 64)
    b.axis_scale = w
    compare(b, run_gpu(b, force_schedule=schedule))


@pytest.mark.parametrize("mode,k,iters", [(0, 0, 3), (1, 8, 0), (1, 5, 2)])
def test_lloyd_and_knn_under_axis_weights(mode, k, iters):
    b = workloads.random_batch(710 + 3 * mode + iters, [40, 300, 2000, 30000], 32, assign_mode=mode, k=k,
                               lloyd_iters=iters, charge_col=0)
    b.axis_scale = TIME_SCALE
    compare(b, run_gpu(b))


def test_workload_shapes_under_a_time_scale():
    for name in ("c1", "c4"):
        b = workloads.make_workload(name)
        b.axis_scale = TIME_SCALE
        compare(b, run_gpu(b))


def test_unit_weights_give_the_same_bits():
    b = workloads.random_batch(720, [50, 500, 5000], 32, lloyd_iters=1, charge_col=0)
    a = run_gpu(b)
    u = run_gpu(b, axis_scale=(1.0, 1.0, 1.0, 1.0))
    for key in a:
        np.testing.assert_array_equal(a[key], u[key], err_msg=key)


def test_standalone_calls_under_axis_weights():
    b = workloads.random_batch(721, [3, 200, 1500], 16)
    c, f, o, _ = to_dev(b)
    w = np.array(TIME_SCALE, np.float32)
    idx = oracle.fps(b.coords, b.offsets, b.K, axis_scale=w)
    cents = np.where(idx[..., None] >= 0, b.coords[np.maximum(idx, 0)], 0).astype(np.float32)
    valid = np.minimum(b.sizes(), b.K).astype(np.int32)
    cd = torch.from_numpy(cents).cuda()
    got = fps.fps_assign(c, o, cd, axis_scale=TIME_SCALE).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.assign(b.coords, b.offsets, cents, b.K, valid=valid, axis_scale=w))
    got = fps.fps_knn(c, o, cd, 6, axis_scale=TIME_SCALE).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.knn(b.coords, b.offsets, cents, b.K, 6, valid=valid, axis_scale=w))
    tok = torch.from_numpy(oracle.assign(b.coords, b.offsets, cents, b.K, valid=valid, axis_scale=w)).cuda()
    gc, gt = fps.lloyd_refine(c, f, o, cd.clone(), tok.clone(), 2, charge_col=0, axis_scale=TIME_SCALE)
    want_c, want_t = oracle.lloyd(b.coords, b.feats, b.offsets, b.K, 2, cents,
                                  tok.cpu().numpy(), charge_col=0, axis_scale=w)
    big = np.repeat(b.sizes() > b.K, b.sizes())
    err = np.abs(gc.cpu().numpy().astype(np.float64) - want_c)
    assert np.all(err <= 1e-5 * np.abs(want_c) + 1e-6)
    # the labels are exactly the nearest of the GPU's own refined centroids
    np.testing.assert_array_equal(gt.cpu().numpy()[big], oracle.assign(b.coords, b.offsets, gc.cpu().numpy(),
                                                                        b.K, valid=valid, axis_scale=w)[big])
