"""Host-side dispatch and tile planning (ll_plan): no GPU needed.

The pins are measured on one B200 (148 SMs):
- Dispatch crossovers, from ``python bench.py --suite crossover --rank 64
  --steps 10 --warmup 3`` (every variant against M on the K = 4096,
  N = 16384 family, L2 flushed between calls): the streaming kernel is the
  fastest up to 64 tokens (29.7 us at M = 1 and 64, against 39.9 us and
  more for the others), the CTA-pair kernel from 96 to 256 tokens (37.9 to
  39.9 us, against 40.0 to 68.6 us for the 128 x 128 kernel and 42.0 to
  44.1 us for the one-CTA fused kernel), the one-CTA fused kernel above.
- Tile plans, from ``python bench.py --workload <name> --steps 50
  --warmup 5`` per configuration: 256-token tiles with one down-projection
  split at the attention, FFN and sweep shapes (forward 42.9 us for the
  attention projection against 47.7 us for the previous 224-token plan).
- The FP8-operand two-term kernel above 256 tokens where N >= 2K, or
  N >= K with M >= 4096, from forward times measured per variant with L2
  flushed between calls (us, exact-widening / two-term): 3630 x 2048 ->
  8192 122 / 101; 1024 x 4096 -> 16384 122 / 108; 4096 x 4096 -> 4096
  124 / 118; 1024 x 4096 -> 4096 40 / 63; 3630 x 2048 -> 2048 42 / 54;
  3630 x 8192 -> 2048 118 / 169; 9800 x 16384 -> 4096 1071 / 1112.

The properties hold for every plan the library can make.
"""
import itertools

import pytest

import rank_fp8_residual_b200 as ll

SMS = 148


@pytest.mark.parametrize("N,K,r,M,kernel", [
    (2048, 2048, 32, 3630, ll.LL_VARIANT_TC),           # attention projection
    (8192, 2048, 64, 3630, ll.LL_VARIANT_FP8_SPLIT),    # FFN up
    (2048, 8192, 64, 3630, ll.LL_VARIANT_TC),           # FFN down
    (16384, 4096, 64, 8192, ll.LL_VARIANT_FP8_SPLIT),   # sweep point
    (4096, 4096, 64, 1024, ll.LL_VARIANT_TC),           # sweep point, N = K, M < 4096
    (4096, 4096, 64, 4096, ll.LL_VARIANT_FP8_SPLIT),    # sweep point, N = K, M >= 4096
    (4096, 16384, 64, 9800, ll.LL_VARIANT_TC),          # README benchmark w2
])
def test_large_m_plans(N, K, r, M, kernel):
    got, bt, ks = ll.ll_plan(N, K, r, M, SMS)
    assert got == kernel
    assert bt == 256
    if kernel == ll.LL_VARIANT_TC:
        assert ks == 1


@pytest.mark.parametrize("M", [2, 16, 33, 64])
def test_small_batch_streams(M):
    kernel, bt, ks = ll.ll_plan(16384, 4096, 512, M, SMS)
    assert kernel == ll.LL_VARIANT_STREAM
    assert bt == (M + 15) // 16 * 16
    assert 1 <= ks <= 8


def test_one_token_runs_the_gemv_when_x_fits():
    """Measured at K = 4096, N = 16384, r = 512 (python bench.py configs;
    forward us, L2 flushed): one token 29.7 on the GEMV against 31.8 on the
    streaming kernel; two tokens 33.8 against 31.7."""
    assert ll.ll_plan(16384, 4096, 512, 1, SMS)[:2] == (ll.LL_VARIANT_GEMV, 1)
    assert ll.ll_plan(1024, 49152, 64, 1, SMS)[0] == ll.LL_VARIANT_GEMV      # 96 KB of x fits
    assert ll.ll_plan(1024, 65536, 64, 1, SMS)[0] == ll.LL_VARIANT_STREAM    # 128 KB does not


def test_auto_crossovers():
    for M, want in [(64, ll.LL_VARIANT_STREAM), (65, ll.LL_VARIANT_TC_PAIR), (256, ll.LL_VARIANT_TC_PAIR),
                    (257, ll.LL_VARIANT_FP8_SPLIT), (4096, ll.LL_VARIANT_FP8_SPLIT)]:
        assert ll.ll_plan(16384, 4096, 64, M, SMS)[0] == want, M
    for M, want in [(257, ll.LL_VARIANT_TC), (4095, ll.LL_VARIANT_TC), (4096, ll.LL_VARIANT_FP8_SPLIT)]:
        assert ll.ll_plan(4096, 4096, 64, M, SMS)[0] == want, M
    for M in (257, 3630, 16384):
        assert ll.ll_plan(2048, 8192, 64, M, SMS)[0] == ll.LL_VARIANT_TC, M


def test_forced_variants():
    for M in (1, 100, 3000):
        assert ll.ll_plan(4096, 4096, 64, M, SMS, ll.LL_VARIANT_TC)[0] == ll.LL_VARIANT_TC
        assert ll.ll_plan(4096, 4096, 64, M, SMS, ll.LL_VARIANT_TC_PAIR)[0] == ll.LL_VARIANT_TC_PAIR
        assert ll.ll_plan(4096, 4096, 64, M, SMS, ll.LL_VARIANT_SMALL)[0] == ll.LL_VARIANT_SMALL
        want = ll.LL_VARIANT_STREAM if M <= 64 else ll.LL_VARIANT_SMALL
        assert ll.ll_plan(4096, 4096, 64, M, SMS, ll.LL_VARIANT_STREAM)[0] == want


def test_plan_properties():
    Ns = (256, 2048, 16384)
    Ks = (256, 4096, 8192)
    rs = (0, 16, 32, 64, 200, 512)
    Ms = (1, 63, 64, 65, 128, 129, 256, 257, 1000, 3630, 16384)
    for N, K, r, M in itertools.product(Ns, Ks, rs, Ms):
        kernel, bt, ks = ll.ll_plan(N, K, r, M, SMS)
        assert kernel in (ll.LL_VARIANT_TC, ll.LL_VARIANT_TC_PAIR, ll.LL_VARIANT_STREAM, ll.LL_VARIANT_FP8_SPLIT,
                          ll.LL_VARIANT_GEMV)
        if kernel == ll.LL_VARIANT_GEMV:
            assert M == 1 and bt == 1 and ks == 1
            continue
        if kernel == ll.LL_VARIANT_FP8_SPLIT:
            assert bt == 256 and M > 256 and (N >= 2 * K or (N >= K and M >= 4096))
        elif kernel == ll.LL_VARIANT_TC:
            assert bt % 32 == 0 and 128 <= bt <= 256
        elif kernel == ll.LL_VARIANT_TC_PAIR:
            assert bt % 32 == 0 and 32 <= bt <= 256
        else:
            assert bt == (M + 15) // 16 * 16 and bt <= 64
        n_kstep = (K + 63) // 64
        if r == 0:
            assert ks == 1
        else:
            assert 1 <= ks <= min(8, n_kstep)
            if kernel == ll.LL_VARIANT_TC and M > 128 and ks > 1:
                r_pad = (r + 31) // 32 * 32
                rc = min(r_pad, 256)
                ctas = (M + 127) // 128 * ((r_pad + rc - 1) // rc) * ks
                assert ctas <= SMS


def test_plan_rejects_bad_arguments():
    with pytest.raises(ll.LLError):
        ll.ll_plan(100, 4096, 64, 64, SMS)        # N % 8
    with pytest.raises(ll.LLError):
        ll.ll_plan(4096, 100, 64, 64, SMS)        # K % 16
    with pytest.raises(ll.LLError):
        ll.ll_plan(4096, 4096, 64, 0, SMS)        # M < 1
    with pytest.raises(ll.LLError):
        ll.ll_plan(4096, 4096, 64, 64, 1)         # num_sms < 2
    with pytest.raises(ll.LLError):
        ll.ll_plan(4096, 4096, 64, 64, SMS, 9)    # unknown variant
    for v in (ll.LL_VARIANT_FP8_SPLIT, ll.LL_VARIANT_FP8_ACT):
        assert ll.ll_plan(4096, 4096, 64, 100, SMS, v)[0] == v
    with pytest.raises(ll.LLError):
        ll.ll_plan(4096, 4096, 513, 64, SMS)      # r > 512
