"""Host-side test of the paged optimizer's placement under a memory spike
(intvml.com "DL0087 QLoRA", component (5) "Paged Optimizers": the optimizer
state moves to host RAM when device memory runs short and comes back
afterwards). The spike is made on the host: a sequence of free-device-memory
readings, as cudaMemGetInfo would return them before each step while another
allocation (a long-sequence activation burst under gradient checkpointing)
comes and goes, is fed to the library's policy function; no GPU is used.
"""
import pytest

from bit_quantized_lora_blockwise_b200 import binding

GB = 1 << 30


@pytest.fixture(scope="module")
def lib():
    return binding.load()


def _run(readings, state, reserve, start=0):
    where, trace = start, []
    for free in readings:
        where = binding.paged_adamw_placement(free, state, reserve, where)
        trace.append(where)
    return trace


def test_spike_pages_out_and_back(lib):
    state, reserve = 2 * GB, 4 * GB
    # plenty free, a spike leaves 1 GB, the spike ends
    readings = [100 * GB, 90 * GB, 1 * GB, 1 * GB, 3 * GB, 5 * GB, 6 * GB, 80 * GB]
    assert _run(readings, state, reserve) == [0, 0, 1, 1, 1, 1, 0, 0]


def test_hysteresis_needs_room_for_the_state(lib):
    state, reserve = 2 * GB, 4 * GB
    # on the host: back only when the state and the reserve both fit
    assert binding.paged_adamw_placement(6 * GB - 1, state, reserve, 1) == 1
    assert binding.paged_adamw_placement(6 * GB, state, reserve, 1) == 0
    # on the device: stays while free >= reserve (its own pages are already counted as used)
    assert binding.paged_adamw_placement(4 * GB, state, reserve, 0) == 0
    assert binding.paged_adamw_placement(4 * GB - 1, state, reserve, 0) == 1


def test_no_reserve_never_pages_out(lib):
    assert _run([0, 1, 50 * GB], 2 * GB, 0) == [0, 0, 0]


def test_oscillating_pressure_does_not_flap(lib):
    state, reserve = 8 * GB, 4 * GB
    readings = [3 * GB, 5 * GB, 3 * GB, 5 * GB, 11 * GB, 12 * GB, 3 * GB]
    assert _run(readings, state, reserve) == [1, 1, 1, 1, 1, 0, 1]
