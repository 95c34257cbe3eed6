"""CPU checks of the C ABI: the library loads, exports every function that
include/moe.h declares, and rejects invalid arguments on the host before any
CUDA call."""
import ctypes

import pytest

import top_routing_grouped_gemv_b200 as moe


@pytest.fixture(scope="module")
def lib():
    moe.build()
    return moe.load()


def test_header_declares_the_stage_entry_points():
    names = set(moe.header_functions())
    for n in ("moe_router_topk", "moe_permute", "moe_grouped_ffn", "moe_unpermute_combine",
              "moe_forward", "moe_plan_create", "moe_workspace_size", "moe_read_device_status"):
        assert n in names


def test_library_exports_every_header_symbol(lib):
    missing = [n for n in moe.header_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_struct_layouts_match_header():
    assert ctypes.sizeof(moe.LayerDesc) == 32
    assert ctypes.sizeof(moe.LayerWeights) == 72


def test_status_strings(lib):
    for code in range(7):
        assert lib.moe_status_string(code)


def _create(lib, N=64, d=64, E=8, K=2, F=64, dtype=moe.MOE_BF16, act=moe.ACT_SWIGLU,
            quant=moe.QUANT_NONE, w1=0x1000, w3=0x2000, w2=0x3000, w_r=0x4000, w_mx=None,
            w_gs=None):
    desc = moe.LayerDesc(N, d, E, K, F, dtype, act, quant)
    w = moe.LayerWeights(w_r, None, w1, w3, w2, 1.0, None, w_mx, w_gs)
    h = ctypes.c_void_p()
    rc = lib.moe_plan_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(h))
    if rc == 0:
        lib.moe_plan_destroy(h)
    return rc


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), 1), (dict(K=0), 1), (dict(K=9, E=16), 1), (dict(K=4, E=2), 1),
    (dict(E=257), 1), (dict(d=65536), 1), (dict(F=70000), 1),
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None), 2),   # e4m3 needs per-tensor
    (dict(quant=moe.QUANT_PER_TENSOR), 2),                                 # per-tensor needs e4m3
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None,
          quant=moe.QUANT_PER_CHANNEL), 1),                                # per-channel needs scales
    (dict(quant=7), 1),                                                    # mode 7 is per call
    (dict(quant=4, w_gs=0x6000), 2), (dict(quant=5, w_gs=0x6000), 2),      # group, block need e4m3
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None,
          quant=moe.QUANT_PER_GROUP), 1),                                  # group needs its scales
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None, d=192,
          quant=moe.QUANT_PER_BLOCK, w_gs=0x6000), 1),                     # d not a multiple of 128
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None,
          quant=moe.QUANT_PER_TENSOR, w_gs=0x6000), 1),                    # scales without the mode
    (dict(quant=3), 2),                                                    # per-token is per call
    (dict(quant=moe.QUANT_MX, w_mx=0x5000), 2),                            # MX needs e4m3
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None,
          quant=moe.QUANT_MX), 1),                                         # MX needs its scales
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None, d=48,
          quant=moe.QUANT_MX, w_mx=0x5000), 1),                            # d not a multiple of 32
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None, d=32800,
          quant=moe.QUANT_MX, w_mx=0x5000), 1),                            # d above 32768
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_NONE, w3=None, w2=None,
          quant=moe.QUANT_PER_TENSOR, w_mx=0x5000), 1),                    # scales without MX
    (dict(dtype=moe.MOE_E4M3, act=moe.ACT_SWIGLU, quant=moe.QUANT_PER_TENSOR), 2),
    (dict(dtype=moe.MOE_BF16, act=moe.ACT_RELU, w3=None), 2),
    (dict(w3=None), 1),                                                    # SwiGLU needs w3
    (dict(act=moe.ACT_NONE), 1),                                           # NONE takes no w2/w3
    (dict(w1=0x1008), 1),                                                  # misaligned weights
    (dict(d=60), 1),                                                       # 120-byte rows
])
def test_plan_validation_rejects(lib, kw, code):
    assert _create(lib, **kw) == code


def test_null_arguments(lib):
    assert lib.moe_plan_create(None, None, None) == 1
    assert lib.moe_plan_destroy(None) == 1
    assert lib.moe_workspace_size(None, None) == 1
    assert lib.moe_forward(None, None, None, None, 0, None) == 1
    assert lib.moe_last_launch_count(None) == -1
    # the quant-mode calls refuse a null plan before anything else
    assert lib.moe_forward_routed_mx(None, None, None, None, None, None, None, 0, None) == 1
    assert lib.moe_permute_mx(None, None, None, None, None, None, None, None, None, None, None, 0,
                              None) == 1
    assert lib.moe_grouped_ffn_mx(None, None, None, None, None, None, 0, None) == 1
    assert lib.moe_forward_routed_group_scales(None, None, 1.0, None, None, None, None, None, None,
                                               0, None) == 1
    assert lib.moe_grouped_ffn_group_scales(None, None, 1.0, None, None, None, None, None, 0,
                                            None) == 1


def test_binding_refuses_two_weight_scale_modes():
    """The Python plan takes one weight scale mode (the C ABI has one quant
    field): two kinds of scales in the weights dict are an error before the
    library is asked."""
    with pytest.raises(ValueError, match="one weight scale mode"):
        moe.Plan(16, 64, 4, 2, 32, "e4m3", "none",
                 {"w1": None, "w_mx_scales": object(), "w_group_scales": object()})
