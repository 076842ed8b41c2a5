"""The roofline numerators of the benchmark: algorithmic bytes per decode launch and per quantised element.

They follow from the record layout (include/kvarn.h): per block of 128 tokens and D = 128 channels, 2-bit codes
(4096 B), binary16 (s, m) per token and 32-channel group (2048 B), binary16 r per token (256 B) and c per channel
(256 B).  These checks tie the benchmark's constants to the library's own record size and to the per-token figure
of 104 B (K and V) at D = 128."""
import importlib.util
import os

from bit_kv_cache_token_b200 import kvarn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_record_size_matches_library():
    rb = kvarn.record_bytes(kvarn.Config(1, 1, 128, 1))
    assert rb == 4096 + 2048 + 256 + 256 == 6656
    assert 2 * rb / 128 == 104  # K + V bytes per cached token and kv head


def test_decode_bytes_at_32705_tokens():
    b = _bench()
    assert (b.S, b.HKV, b.HQ, b.D) == (8, 8, 32, 128)
    full = 255 * 128 * 104 * 8 * 8          # 255 full blocks of K and V records
    tail = 65 * 2 * 128 * 2 * 8 * 8         # 65 bf16 tail tokens of K and V
    qo = 8 * 32 * 128 * (2 + 4)             # bf16 q in, fp32 out
    assert b.decode_bytes(32705) == full + tail + qo == 219_578_368


def test_decode_bytes_edge_cases():
    b = _bench()
    assert b.decode_bytes(0) == 8 * 32 * 128 * 6              # only q and out
    assert b.decode_bytes(128) - b.decode_bytes(0) == 8 * 8 * 2 * 6656
    assert b.decode_bytes(127) - b.decode_bytes(0) == 8 * 8 * 127 * 2 * 128 * 2


def test_quant_bytes_per_element():
    b = _bench()
    n = 32 * 32 * 8 * 8192 * 128 * 2                           # Llama-3-8B-shaped bulk workload, K and V
    assert b.quant_bytes(n) / n == 2.40625
    assert b.quant_bytes(n) == 41_339_060_224
