"""The bench's algorithmic byte and FLOP counts (CPU only): the per-unit sizes
and the totals the roofline fractions divide by, against the numbers stated
for the workload (hidden 1280, intermediate 896, 64 routed + 2 shared experts,
top-6, 12 layers, vocabulary 129,280)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_unit_sizes():
    assert bench.EXPERT_W_BYTES == 3 * 896 * 1280 * 2 == 6_881_280  # gate, up, down in bf16
    assert bench.ROUTER_W_BYTES == 64 * 1280 * 2 == 163_840
    assert bench.LM_HEAD_BYTES == 129_280 * 1280 * 2 == 330_956_800


def test_decode_step_bytes():
    # every expert touched at 128 tokens: 12 x (router + 66 experts) + the LM head
    full = bench.step_weight_bytes([64] * 12)
    assert full == 12 * (163_840 + 66 * 6_881_280) + 330_956_800 == 5_782_896_640
    # the time this takes at the nominal 8 TB/s and at the measured 6,545.3 GB/s copy rate
    assert abs(full / 8e12 * 1e3 - 0.7229) < 1e-4
    assert abs(full / 6545.3e9 * 1e3 - 0.8835) < 1e-4
    # untouched experts cost nothing; the shared ones always count
    assert bench.step_weight_bytes([0] * 12) == 12 * (163_840 + 2 * 6_881_280) + 330_956_800
    assert bench.step_weight_bytes([21] * 12) < full


def test_prefill_and_skew_flop():
    T = 32 * 1156
    routed, shared, router = 2 * 6 * T * 3 * 896 * 1280, 2 * 2 * T * 3 * 896 * 1280, 2 * T * 64 * 1280
    assert bench.PREFILL_T == T == 36_992
    assert bench.PREFILL_FLOP == routed + shared + router
    assert abs(routed / 1e12 - 1.527) < 1e-3 and abs(shared / 1e12 - 0.509) < 1e-3
    assert abs(bench.PREFILL_FLOP / 1e12 - 2.043) < 1e-3
    assert bench.SKEW_FLOP == 2 * 8 * 4096 * 3 * 896 * 1280 + 2 * 4096 * 64 * 1280


def test_attention_bytes():
    # B = 32, K = 3, L = 2,048: weights 4 H^2, keys and values of L + 4 positions
    # read, the 4 new rows' keys and values written, input and output, bf16
    assert bench.attention_bytes(2048) == (4 * 1280 * 1280 + 32 * 2052 * 2560 + 32 * 4 * 2560
                                           + 2 * 128 * 1280) * 2 == 350_617_600
    # one chunk launch: every visible key and value, the rotated queries, the
    # fp32 partials of 9 chunks of 256 positions (max, exp-sum, 128 values)
    assert bench.attention_chunk_bytes(2048) == 32 * 2052 * 2560 * 2 + 32 * 4 * 1280 * 2 + 32 * 10 * 9 * 4 * 130 * 4
