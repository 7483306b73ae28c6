"""The cluster schedules' bounded exchange wait, made to run out on purpose.

Every FPS step of an 8- or 16-CTA cluster waits on an mbarrier for the other
CTAs' candidates; each wait polls a bounded number of times.  A host-side
test setting (``fps_set_exchange_test``) shortens the limit and makes one CTA
of every cluster skip its post in the first exchange of each event, so that
every wait of that round runs out.  The launch must end by itself, report
FPS_DEV_EXCHANGE_TIMEOUT through the device status word, and leave the CUDA
context usable: the same batch and the tiny workload then match the oracle
again.  Nothing faults or hangs: the waits are bounded and the kernel returns
on its own; the skipped post is a flag read on the host side of the launch.
"""
import pytest

import workloads
from parity import compare, run_gpu, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import farthest_point_sampling_b200 as fps  # noqa: E402

FPS_DEV_EXCHANGE_TIMEOUT = 5


@pytest.mark.parametrize("schedule,sizes", [(3, [9000, 130, 20000, 40]), (4, [120000, 5000])])
def test_exchange_timeout_is_reported_and_the_context_stays_usable(schedule, sizes):
    lib = fps.load_library()
    b = workloads.random_batch(610 + schedule, sizes, 64)
    c, f, o, _ = to_dev(b)
    try:
        lib.fps_set_exchange_test(1024, 1)  # 1024 polls per wait; CTA 1 skips its first post
        with pytest.raises(fps.FpsError) as err:
            fps.fps_tokenize(c, f, o, K=b.K, force_schedule=schedule, check_device=True)
        assert getattr(err.value, "detail", None) == FPS_DEV_EXCHANGE_TIMEOUT
    finally:
        lib.fps_set_exchange_test(0, -1)
    torch.cuda.synchronize()
    # the context still works: the same batch on the same schedule, then the tiny workload
    compare(b, run_gpu(b, force_schedule=schedule))
    b0 = workloads.make_workload("c0")
    compare(b0, run_gpu(b0))


def test_default_exchange_setting_reports_nothing():
    lib = fps.load_library()
    lib.fps_set_exchange_test(0, -1)
    b = workloads.random_batch(615, [30000, 300], 32)
    compare(b, run_gpu(b, force_schedule=3))  # run_gpu checks the device status word
