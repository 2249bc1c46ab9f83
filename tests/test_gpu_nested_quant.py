"""GPU parity of the 4-bit quantize and the nested 4-bit state against the oracle (bit-exact),
through the C ABI. The encode is the reading stated in include/bbc.h (the pages give only the
decode, "Fuse nested 4-bit scale reconstruction on SM103")."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import DTYPES, assert_bits_equal, to_host

pytestmark = pytest.mark.gpu
NAMES = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}
NF4 = oracle.normal_float_codebook(4)
FP4 = synthetic.fp4_table()
G8 = synthetic.general8_table()


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def check_q4(bbc, x_host, bs, code4, x_dev=None, codes_buf=None, what=""):
    dt = NAMES[x_host.dtype]
    n = x_host.numel()
    ref_c, ref_a = oracle.quantize_4bit(to_host(x_host), dt, bs, code4)
    codes, absmax = bbc.quantize_4bit(x_host.cuda() if x_dev is None else x_dev, bs,
                                      torch.from_numpy(code4).cuda(), codes=codes_buf)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(absmax)[:ref_a.size], ref_a, f"q4 absmax {what} bs={bs} {dt}")
    assert_bits_equal(to_host(codes)[:(n + 1) // 2], ref_c, f"q4 codes {what} bs={bs} {dt}")


@pytest.mark.parametrize("table", ["nf4", "fp4"])
@pytest.mark.parametrize("bs", [32, 64, 128, 256, 512, 1024, 2048, 4096])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_quantize_4bit_matrix(bbc, table, bs, dt):
    n = 3 * 4096 * 5 + 37                   # several CTA chunks, a partial block, odd n
    x = synthetic.weights(n, std=0.02, seed=bs, dtype=DTYPES[dt], outlier_frac=0.001)
    check_q4(bbc, x, bs, NF4 if table == "nf4" else FP4, what=table)


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_quantize_4bit_ragged_and_unaligned(bbc, dt):
    for n in [1, 2, 15, 16, 17, 33, 1000, 4095, 4097, 65537]:
        check_q4(bbc, synthetic.weights(n, std=1.0, seed=n, dtype=DTYPES[dt]), 64, NF4, what=f"n={n}")
    n = 4096 * 3 + 21
    x = synthetic.weights(n + 1, std=0.5, seed=3, dtype=DTYPES[dt])
    buf = torch.zeros((n + 1) // 2 + 1, dtype=torch.uint8, device="cuda")
    check_q4(bbc, x[1:].contiguous(), 128, NF4, x_dev=x.cuda()[1:], codes_buf=buf[1:], what="offsets")
    assert int(buf[0]) == 0


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_quantize_4bit_special_blocks(bbc, dt):
    bs = 64
    rng = np.random.default_rng(8)
    x = (rng.standard_normal(bs * 12) * 0.1).astype(np.float32)
    x[0:bs] = 0.0                                      # zero block
    x[bs + 3] = np.nan                                 # one NaN
    x[2 * bs:3 * bs] = np.nan                          # all NaN
    x[3 * bs + 5] = np.inf
    x[4 * bs + 7] = -np.inf
    x[5 * bs:6 * bs] *= 1e-35                          # tiny (below the 1e-8 clamp)
    x[6 * bs + 1] = 3e38                               # huge (f32 only; inf in 16-bit types)
    x[7 * bs:8 * bs] = 1e-42                           # fp32 subnormals
    check_q4(bbc, torch.from_numpy(x).to(DTYPES[dt]), bs, NF4, what="special")
    check_q4(bbc, torch.from_numpy(x).to(DTYPES[dt]), bs, FP4, what="special fp4")


def check_nested(bbc, x, bs, code2=G8, what=""):
    dt = NAMES[x.dtype]
    ref = oracle.quantize_4bit_nested(to_host(x), dt, bs, NF4, code2)
    codes, q, a2, off = bbc.quantize_4bit_nested(x.cuda(), bs, torch.from_numpy(NF4).cuda(),
                                                 torch.from_numpy(code2).cuda())
    torch.cuda.synchronize()
    n = x.numel()
    assert_bits_equal(to_host(codes)[:(n + 1) // 2], ref[0], f"nested codes {what}")
    assert_bits_equal(to_host(q)[:ref[1].size], ref[1], f"absmax_q {what}")
    assert_bits_equal(to_host(a2)[:ref[2].size], ref[2], f"absmax2 {what}")
    assert_bits_equal(to_host(off), np.array([ref[3]], np.float32), f"offset {what}")
    return codes, q, a2, off, ref


def test_nested_state_c3_size(bbc):
    """4096x11008 bf16 weights ~ N(0, 0.02), outer blocksize 64: 704,512 outer blocks (344 binary64
    partial chunks, 2,752 inner groups); the nested dequant of the GPU state matches the oracle's."""
    x = synthetic.weights(4096 * 11008, std=0.02, seed=3, dtype=torch.bfloat16)
    codes, q, a2, off, ref = check_nested(bbc, x, 64, what="c3")
    n = x.numel()
    y = bbc.dequantize_4bit_nested(codes, q, torch.from_numpy(G8).cuda(), a2, float(off.item()),
                                   torch.from_numpy(NF4).cuda(), n, 64, torch.bfloat16)
    torch.cuda.synchronize()
    ref_y = oracle.nested_dequantize(ref[0], ref[1], G8, ref[2], float(ref[3]), NF4, n, 64, 256, "bf16")
    assert_bits_equal(to_host(y)[:n], ref_y, "nested round trip bf16")


@pytest.mark.parametrize("bs", [32, 4096])
@pytest.mark.parametrize("dt", ["f16", "f32"])
def test_nested_state_blocksizes(bbc, bs, dt):
    n = bs * 256 * 3 + bs * 5 + 11          # partial inner group and partial outer block
    check_nested(bbc, synthetic.weights(n, std=0.05, seed=bs + 1, dtype=DTYPES[dt]), bs, what=f"bs={bs} {dt}")


def test_nested_state_unsorted_code2(bbc):
    """A General8 table that is not ascending takes the verbatim nearest-entry rule."""
    perm = np.random.default_rng(9).permutation(256)
    x = synthetic.weights(64 * 256 * 2 + 3, std=0.02, seed=12, dtype=torch.bfloat16)
    check_nested(bbc, x, 64, code2=np.ascontiguousarray(G8[perm]), what="shuffled code2")


def test_nested_state_small_and_constant(bbc):
    for n in [1, 63, 64, 65, 64 * 2048 + 1]:
        check_nested(bbc, synthetic.weights(n, std=1.0, seed=n, dtype=torch.float32), 64, what=f"n={n}")
    # every outer absmax equal: absmax2 = 0, the divisor clamps to 1e-8
    x = torch.ones(64 * 300, dtype=torch.float32) * 0.25
    check_nested(bbc, x, 64, what="constant")


@pytest.mark.parametrize("table", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_every_16bit_quotient_4bit(bbc, table, dt):
    """Every value of the 16-bit type in [-d, d] as a numerator for several block maxima d
    (blocksize 32: the block's first element is d), so every quotient these d produce, on and
    beside each threshold of the table, is decided by the kernel's exact search."""
    code4 = NF4 if table == "nf4" else FP4
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    widen = oracle.bf16_bits_to_f32 if dt == "bf16" else oracle.f16_bits_to_f32
    narrow = oracle.f32_to_bf16_bits if dt == "bf16" else oracle.f32_to_f16_bits
    vals = widen(bits)
    blocks = []
    for d_req in (1.0, 0.7373, 3.25e-3, 1234.5):
        d_bits = narrow(np.array([d_req], np.float32))[0]
        d = widen(np.array([d_bits], np.uint16))[0]
        xs = bits[np.isfinite(vals) & (np.abs(vals) <= d)]
        for i in range(0, xs.size, 31):
            blk = np.zeros(32, np.uint16)
            blk[0] = d_bits
            blk[1:1 + xs[i:i + 31].size] = xs[i:i + 31]
            blocks.append(blk)
    x = np.concatenate(blocks)
    check_q4(bbc, torch.from_numpy(x.view(np.int16)).view(DTYPES[dt]), 32, code4, what=f"every {dt} quotient")


def test_nested_state_two_tree_levels(bbc):
    """4,198,405 outer blocks (blocksize 32): the offset tree takes two level launches (2,051
    first-level nodes, an odd count, then 2) before the root, which reads the second node
    buffer."""
    nbo = 2048 * 2048 + 2048 * 2 + 5
    x = synthetic.weights(32 * nbo - 7, std=0.02, seed=77, dtype=torch.bfloat16)
    check_nested(bbc, x, 32, what="two tree levels")


def _quotients(x_host, bs):
    """The scaled values the General8 search sees for this input (used only to place table
    entries on and beside them; the expected state still comes from the oracle)."""
    _, absmax = oracle.quantize_4bit(to_host(x_host), NAMES[x_host.dtype], bs, NF4)
    c = absmax - oracle.absmax_offset(absmax)
    pad = (-c.size) % 256
    d = np.abs(np.concatenate([c, np.zeros(pad, np.float32)])).reshape(-1, 256).max(axis=1)
    d = np.maximum(d, np.float32(1e-8)).astype(np.float32)
    return (c / np.repeat(d, 256)[:c.size]).astype(np.float32)


@pytest.mark.parametrize("kind", ["straddle", "decade", "scaled"])
def test_nested_compression_switch_point_tables(bbc, kind):
    """Tables in the compression's fast form (finite, strictly ascending, neighbouring gaps within
    a factor 2^20): entry pairs straddling 48 of the quotients the input produces, so that switch
    points fall on and one ulp beside them; a table built by decades from 1e-7 to 1; and the
    stand-in table scaled by 0.9, so that the quotients +-1 of every group's largest block lie
    beyond both end entries."""
    from tests.test_model_compression_switch_points import decade_table, fast_form_ok
    bs = 64
    x = synthetic.weights(bs * 256 * 5 + bs * 9 + 5, std=0.02, seed=33, dtype=torch.float32)
    if kind == "straddle":
        xn = _quotients(x, bs)
        rng = np.random.default_rng(43)
        picks = np.unique(rng.choice(xn[np.abs(xn) < 0.95], 48, replace=False))
        delta = (np.abs(picks) * 1e-3 + 1e-7).astype(np.float32)
        lo, hi = (picks - delta).astype(np.float32), (picks + delta).astype(np.float32)
        # symmetric pairs put the switch point one ulp above the pick (the tie stays with the
        # lower entry); lowering every other lower entry by two ulps puts it on the pick
        lo[1::2] = np.nextafter(np.nextafter(lo[1::2], np.float32(-2)), np.float32(-2))
        pairs = np.concatenate([lo, hi]).astype(np.float32)
        fill = np.linspace(-1, 1, 256 - pairs.size).astype(np.float32)
        table = np.sort(np.concatenate([pairs, fill])).astype(np.float32)
    elif kind == "decade":
        table = decade_table()
    else:
        table = (G8 * np.float32(0.9)).astype(np.float32)
    assert table.size == 256 and fast_form_ok(table)
    check_nested(bbc, x, bs, code2=table, what=f"fast form {kind}")


@pytest.mark.parametrize("kind", ["hits", "cluster", "duplicates", "infinite_ends", "all_equal"])
def test_nested_compression_crafted_tables(bbc, kind):
    """Ascending tables placed around the quotients the input produces: entries equal to
    quotients and one ulp beside them (exact and near ties), a dense cluster of 160 entries
    around the median quotient (many entries per bucket of the search), runs of equal entries
    (plateaus of equal distance), infinite end entries, and a table of one repeated value."""
    bs = 64
    x = synthetic.weights(bs * 256 * 5 + bs * 9 + 5, std=0.02, seed=31, dtype=torch.float32)
    xn = _quotients(x, bs)
    rng = np.random.default_rng(41)
    picks = rng.choice(xn, 48, replace=False)
    med = np.float32(np.median(xn))
    if kind == "hits":
        parts = [picks, np.nextafter(picks, np.float32(2)), np.nextafter(picks, np.float32(-2))]
    elif kind == "cluster":
        parts = [np.linspace(med - 2e-4, med + 2e-4, 160, dtype=np.float32), picks]
    elif kind == "duplicates":
        parts = [np.repeat(picks[:20], 4), np.repeat(np.float32(med), 30), picks[20:]]
    elif kind == "infinite_ends":
        parts = [np.array([-np.inf, np.inf], np.float32), picks]
    else:
        parts = [np.full(256, med, np.float32)]
    have = np.concatenate(parts).astype(np.float32)[:256]
    fill = rng.uniform(-1, 1, 256 - have.size).astype(np.float32)
    table = np.sort(np.concatenate([have, fill])).astype(np.float32)
    assert table.size == 256 and np.all(table[:-1] <= table[1:])
    check_nested(bbc, x, bs, code2=table, what=f"crafted {kind}")
