"""Host-side argument validation of every compute entry of the C ABI
(include/mxmoe.h), on the CPU.

For each entry a call whose arguments are all valid on the host is built; on
a machine without a CUDA device that call passes every host check and stops
at the device check with MX_ECUDA.  Each mutation then breaks exactly one
documented requirement (a null pointer, a size that is not a multiple of the
tile or block, a misaligned pointer, an unknown enum value) and must come back
MX_EINVAL: so each rejection is caused by the broken requirement, not by an
earlier one.  No call launches a kernel.
"""
import numpy as np
import pytest
import torch

from fp8_moe_numerics_b200._lib import MX_ECUDA, MX_EINVAL

_BUF = np.zeros(1 << 16, np.uint8)
A = (_BUF.ctypes.data + 255) // 256 * 256          # a 256-byte aligned host address
A1, A4, A8 = A + 1, A + 4, A + 8                    # misaligned for 16-byte requirements

# entry -> (host-valid arguments, [(name of the broken requirement, {arg index: value})])
CASES = {
    "nvfp4_quantize": ((A, 128, 64, 1, A, A, A, 0, None), [
        ("null x", {0: None}), ("negative rows", {1: -1}), ("cols % 16", {2: 40}), ("group_rows 0", {3: 0}),
        ("rows % group_rows", {3: 3}), ("codes misaligned", {4: A8}), ("x misaligned", {0: A1}),
        ("unknown sf_layout", {7: 2}), ("MMA layout rows % 128", {1: 64, 7: 1}),
    ]),
    "mxfp8_requant_transpose_sr": ((A, A, A, 128, 128, 1, 0, None, 1, 2, 16, A, A, 0, None), [
        ("null codes", {0: None}), ("rows % 128", {3: 100}), ("cols % 64", {4: 96}), ("rbits 7", {10: 7}),
        ("unknown in_sf_layout", {6: 3}), ("unknown out_sf_layout", {13: 3}),
        ("group_rows not a tile multiple", {5: 64}), ("out_codes misaligned", {11: A8}),
        ("MMA output cols % 128", {4: 64, 13: 1}),
    ]),
    "mxfp8_quantize": ((A, 128, 128, 0, 1, 2, 16, None, A, A, A, A, 0, None), [
        ("rows % 128", {1: 100}), ("cols % 128", {2: 96}), ("unknown rounding", {3: 2}),
        ("SR with rbits 4", {3: 1, 6: 4}), ("neither form requested", {8: None, 10: None}),
        ("row codes without scales", {9: None}), ("col codes misaligned", {10: A8}),
        ("unknown sf_layout", {12: 5}), ("x misaligned", {0: A8}),
    ]),
    "grouped_gemm_nvfp4": ((A, A, A, A, A, A, A, 1, 128, 128, 256, A, 0, None), [
        ("K % 256", {10: 128}), ("N % 128", {9: 64}), ("M_cap % 128", {8: 100}), ("no experts", {7: 0}),
        ("unknown out_dtype", {12: 3}), ("a_sf misaligned", {1: A4}), ("null seg_offsets", {6: None}),
        ("out misaligned", {11: A8}),
    ]),
    "grouped_gemm_mxfp8": ((0, A, A, A, A, A, 1, 128, 128, 128, A, 0, None), [
        ("unknown mode", {0: 5}), ("K % 128", {9: 64}), ("N % 128", {8: 96}), ("null out", {10: None}),
        ("unknown out_dtype", {11: 7}), ("b_e8m0 misaligned", {4: A4}),
    ]),
    "moe_route": ((A, 16, 2, 4, 640, A, A, A, A, 4096, None), [
        ("capacity below the padded rows", {4: 512}), ("workspace too small", {9: 16}), ("k > 32", {2: 33}),
        ("no experts", {3: 0}), ("M_cap % 128", {4: 600}), ("null workspace", {8: None}),
        # the scan's (E + 1) int64 starts exceed 48 KiB of shared memory at E = 6144 (E * 8 alone does not)
        ("scan shared memory, E = 6144", {3: 6144, 4: 128 * 6144 + 128, 9: 1 << 20}),
    ]),
    "moe_route_aligned": ((A, 16, 2, 4, 256, 1280, A, A, A, A, 4096, None), [
        ("align 64", {4: 64}), ("M_cap % align", {5: 1152}), ("capacity below the padded rows", {5: 1024}),
        ("k 0", {2: 0}), ("null workspace", {9: None}),
    ]),
    "moe_route_static": ((A, 16, 2, 4, 640, A, A, A, None), [
        ("null topk", {0: None}), ("M_cap % 128", {4: 100}), ("k 0", {2: 0}),
        ("beyond the fixed scratch", {1: 1 << 20, 3: 64}), ("null pos", {7: None}),
        ("scan shared memory, E = 6144", {1: 0, 3: 6144, 4: 128 * 6144 + 128}),
    ]),
    "nvfp4_gather_rows": ((A, A, A, A, 2, 128, 64, A, A, A, None), [
        ("cols % 64", {6: 32}), ("M_cap % 128", {5: 100}), ("k 0", {4: 0}), ("sf misaligned", {1: A1}),
        ("out_codes misaligned", {7: A8}), ("null src", {3: None}),
    ]),
    "moe_permute_row_groups": ((A, 4, A, 6, 512, A, None), [
        ("group_bytes % 16", {4: 520}), ("group_bytes 0", {4: 0}), ("null out", {2: None}), ("null table", {5: None}),
        ("in misaligned", {0: A8}), ("out misaligned", {2: A4}), ("negative ngroups_in", {1: -1}),
    ]),
    "swiglu_fwd": ((A, 128, 64, 1, None, A, None), [
        ("F % 8", {2: 12}), ("null h", {0: None}), ("negative rows", {1: -1}), ("a misaligned", {5: A8}),
    ]),
    "swiglu_bwd": ((A, A, 128, 64, 1, None, A, None), [
        ("null da", {1: None}), ("F % 8", {3: 4}), ("dh misaligned", {6: A8}),
    ]),
    "swiglu_nvfp4_quantize": ((A, 128, 64, 1, None, A, A, A, 0, None), [
        ("F % 16", {2: 24}), ("F above 16384", {2: 16 * 1025}), ("unknown sf_layout", {8: 9}),
        ("MMA layout rows % 128", {1: 100, 8: 1}), ("codes misaligned", {5: A8}), ("null outer", {7: None}),
    ]),
    "moe_combine": ((A, A, None, 16, 2, 64, A, None), [
        ("D % 8", {5: 12}), ("k 0", {4: 0}), ("null y", {0: None}), ("out misaligned", {6: A8}),
    ]),
    "moe_dispatch_grad_mxfp8_quantize": ((A, A, None, 16, 2, 128, 128, None, A, A, A, A, 1, None), [
        ("M_cap % 128", {5: 64}), ("D % 128", {6: 64}), ("k 0", {4: 0}), ("dout misaligned", {0: A8}),
        ("null src", {1: None}), ("row codes misaligned", {8: A8}), ("unknown layout", {12: 5}),
    ]),
    "moe_dispatch_grad": ((A, A, A, None, 16, 2, 128, 64, A, None), [
        ("k > 32", {5: 33}), ("D % 8", {7: 4}), ("dy misaligned", {8: A8}), ("negative M_cap", {6: -1}),
    ]),
    "hadamard_s2f6_quantize": ((A, 128, 64, 1, 2, A, A, None), [
        ("cols % 32", {2: 48}), ("negative rows", {1: -1}), ("codes misaligned", {5: A8}), ("null x", {0: None}),
    ]),
    "grouped_gemm_nvfp4_s2f6": ((A, A, A, A, A, A, A, 1, 128, 128, 256, 1, 2, A, A, None), [
        ("K % 256", {10: 128}), ("N % 128", {9: 64}), ("codes misaligned", {13: A8}), ("null e8m0", {14: None}),
        ("M_cap % 128", {8: 64}), ("e8m0 misaligned", {14: A4}),
    ]),
    "moe_combine_s2f6": ((A, A, A, None, 16, 2, 64, 1, 2, A, None), [
        ("D % 32", {6: 48}), ("k 0", {5: 0}), ("out misaligned", {9: A8}), ("null codes", {0: None}),
    ]),
    "nvfp4_quantize_sr": ((A, 128, 64, 1, 1, 1, 2, 16, A, A, A, 0, None), [
        ("cols % 16", {2: 40}), ("unknown rounding", {4: 3}), ("SR with rbits 12", {7: 12}),
        ("group_rows 0", {3: 0}), ("MMA layout rows % 128", {1: 64, 11: 1}), ("x misaligned", {0: A8}),
        ("null outer", {10: None}),
    ]),
    "nvfp4_requant_transpose_sr": ((A, A, A, 256, 64, 1, 0, 2, 1, 1, 1, 2, 16, A, A, A, 0, None), [
        ("cols % 64", {4: 32}), ("rows per expert % 128", {7: 4}), ("rows % experts", {7: 3}),
        ("no experts", {7: 0}), ("unknown rounding", {9: 2}), ("SR with rbits 4", {12: 4}),
        ("unknown out layout", {16: 3}), ("outer-per-expert flag 2", {8: 2}), ("out codes misaligned", {13: A8}),
        ("null out outer", {15: None}), ("out outer misaligned", {15: A1}),
        ("per-row outer scales over two experts", {8: 0}),
        ("more tile rows than the grid's y axis", {3: 65536 * 128, 5: 128, 7: 1}),
    ]),
    "nvfp4_quantize_transpose_segments": ((A, 256, 128, A, 2, 1, 1, 1, 2, 16, A, A, A, 1, None), [
        ("M % 128", {1: 192}), ("C % 64", {2: 96}), ("no experts", {4: 0}), ("per_row 2", {5: 2}),
        ("MMA output C % 128", {2: 64}), ("null seg", {3: None}), ("x misaligned", {0: A8}),
        ("SR with rbits 4", {9: 4}),
    ]),
    "nvfp4_requant_transpose_segments": ((A, A, A, 1, 1, 256, 128, A, 2, 0, 1, 1, 2, 16, A, A, A, 1, None), [
        ("unknown input layout", {3: 4}), ("group_rows 0", {4: 0}), ("M % group_rows", {4: 3}),
        ("codes misaligned", {0: A8}), ("M % 128", {5: 64}), ("out outer misaligned", {16: A1}),
        ("unknown rounding", {10: 5}), ("more tile rows than the grid's y axis", {5: 65536 * 128}),
    ]),
    "grouped_gemm_nvfp4_wgrad": ((A, A, A, A, A, A, A, 2, 512, 128, 256, A, 0, None), [
        ("M_cap % 256", {8: 384}), ("N % 128", {9: 64}), ("K % 128", {10: 64}), ("no experts", {7: 0}),
        ("unknown out_dtype", {12: 2}), ("a_sf misaligned", {1: A4}), ("null out", {11: None}),
        ("null seg", {6: None}),
    ]),
    "nvfp4_quantize_tile16": ((A, 64, 48, 32, A, A, A, None), [
        ("rows % 16", {1: 40}), ("cols % 16", {2: 40}), ("group_rows % 16", {3: 8}), ("rows % group_rows", {3: 48}),
        ("codes misaligned", {4: A8}), ("null sf_tile", {5: None}),
    ]),
}


@pytest.fixture(scope="module")
def mx():
    from fp8_moe_numerics_b200 import build, _lib
    build.build()
    return _lib.lib()


def test_every_compute_entry_has_cases():
    from fp8_moe_numerics_b200._lib import SIGNATURES
    compute = {n for n in SIGNATURES if not n.startswith("mx_")}
    assert compute == set(CASES)
    for name, (base, _) in CASES.items():
        assert len(base) == len(SIGNATURES[name][1]), name


@pytest.mark.parametrize("name", sorted(CASES))
def test_each_broken_requirement_is_rejected_on_the_host(mx, name):
    if torch.cuda.is_available():
        pytest.skip("the host-valid call would reach a launch on a GPU machine")
    base, mutations = CASES[name]
    fn = getattr(mx, name)
    before = mx.mx_kernel_launches()
    assert fn(*base) == MX_ECUDA, "the host-valid call must pass every host check"
    for what, change in mutations:
        args = list(base)
        for i, v in change.items():
            args[i] = v
        assert fn(*args) == MX_EINVAL, (name, what)
    assert mx.mx_kernel_launches() == before


@pytest.mark.parametrize("name", ["moe_route", "moe_route_static"])
def test_empty_routing_accepts_null_token_arrays(mx, name):
    """An empty problem (T = 0) may pass NULL topk and pos, as the header's
    convention says; the call then fails only at the device check here."""
    if torch.cuda.is_available():
        pytest.skip("the host-valid call would reach a launch on a GPU machine")
    args = {"moe_route": (None, 0, 2, 4, 512, A, A, None, A, 4096, None),
            "moe_route_static": (None, 0, 2, 4, 512, A, A, None, None)}[name]
    assert getattr(mx, name)(*args) == MX_ECUDA


def test_route_workspace_size_saturates_instead_of_wrapping(mx):
    size_max = (1 << 64) - 1
    assert mx.mx_route_workspace_bytes(16, 4) == (1 * 4 + 4) * 4      # one chunk histogram + counts
    assert mx.mx_route_workspace_bytes(1 << 62, 1 << 20) == size_max
    assert mx.mx_route_workspace_bytes((1 << 63) - 1, 2) == ((1 << 55) * 2 + 2) * 4   # largest T, no overflow
    assert mx.mx_route_workspace_bytes((1 << 63) - 1, 1 << 10) == size_max
