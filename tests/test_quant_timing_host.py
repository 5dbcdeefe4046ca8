"""Host-side accounting of the standalone act_quant timing module (no device)."""
import pytest

import quant_timing as qt


def test_algorithmic_bytes():
    # 2 bytes read, 1 (E4M3) or 1/2 (E2M1) code byte and 1/32 scale byte per element
    assert qt.algorithmic_bytes("e4m3", 8192, 8192) == 8192 * 8192 * 3.03125
    assert qt.algorithmic_bytes("fp4", 41, 1536) == 41 * 1536 * 2.53125
    with pytest.raises(KeyError):
        qt.algorithmic_bytes("e5m2", 1, 32)


def test_input_copies_exceed_three_l2():
    l2 = 126 * 2 ** 20
    for M, K in ((8192, 8192), (1024, 4096), (41, 1536)):
        n = qt.input_copies(M * K * 2, l2)
        assert 2 <= n <= 64
        assert n * M * K * 2 > 3 * l2 or n == 64
    assert qt.input_copies(8192 * 8192 * 2, l2) == 3


def test_parse_shape():
    assert qt.parse_shape("41x1536") == (41, 1536)
    assert qt.parse_shape("8192X2048") == (8192, 2048)
    for bad in ("0x32", "4x30", "4x"):
        with pytest.raises(ValueError):
            qt.parse_shape(bad)
