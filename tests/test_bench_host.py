"""The benchmark's roofline numerators, recomputed term by term from the storage formats."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gen import CONFIGS  # noqa: E402


def _rec(out_rows, inp, bits):
    # row record: codes, then inp/64 fp16 scales and inp/64 fp16 biases (16-byte padding is 0 at these sizes)
    return out_rows * (inp * bits // 8 + 4 * (inp // 64))


def test_decode_bytes_per_token_layer_35b():
    H, I, E, K, r, P = 2048, 512, 256, 4, 16, 256
    expert = _rec(2 * I, H, 4) + _rec(H, I, 4)
    assert expert == 1_769_472
    shared_lora = 2 * (r * H * 2 + I * r * 2) + (r * I * 2 + H * r * 2)
    router = _rec(E, H, 8)
    shared_gate = _rec(1, H, 8)
    prerouter = P * H * 2 + P * K * 2 + P * 2 + E * P * 2 + E * 2  # W1 token part, K multi-hot columns, b1, W2, b2
    want = K * expert + expert + shared_lora + router + shared_gate + prerouter
    assert want == 10_835_072
    assert bench.token_layer_bytes(CONFIGS[1]) == want


def test_decode_bytes_per_token_layer_8b():
    H, I, E, K, r, P = 2048, 512, 128, 8, 16, 256
    expert = _rec(2 * I, H, 4) + _rec(H, I, 4)
    want = (K + 1) * expert + 2 * (r * H * 2 + I * r * 2) + (r * I * 2 + H * r * 2) + _rec(E, H, 8) + _rec(1, H, 8) \
        + P * H * 2 + P * K * 2 + P * 2 + E * P * 2 + E * 2
    assert want == 17_570_688
    assert bench.token_layer_bytes(CONFIGS[2]) == want


def test_prefill_expert_flops_per_layer():
    T, K, H, I = 3328, 4, 2048, 512
    routed = T * K * (2 * (2 * I) * H + 2 * H * I)
    shared = T * (2 * (2 * I) * H + 2 * H * I)
    assert bench.expert_flops(CONFIGS[3], T) == routed + shared == 104_689_827_840
