"""The parity cases once more against the debug build (GPU required).

libspkv_debug.so holds the same kernels built with SPKV_DEBUG: before a page number read
from a page table is used as an address it is checked against the pool (and query
positions against 0); a failed check latches SPKV_FLAG_INDEX, which spkv_cache_check
reports as SPKV_ERR_INDEX.  On valid states the checks must stay quiet and the results
must still match the oracle: every case below asserts spkv_cache_check == SPKV_OK and
its oracle comparison, with the library calls routed through the debug build.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sparse_decode_attention_spkv_b200 import spkv as S
    from tests import test_gpu_parity as P
    from tests import test_gpu_rethreshold as RT
    from tests import test_gpu_seqsplit as SQ


@pytest.fixture
def debug_build(monkeypatch):
    monkeypatch.setattr(S, "lib", S.open_library(S.DEBUG_LIB_PATH))


@pytest.mark.parametrize("name", ["tiny_f32_one_chunk", "bf16_g4_chunks", "tc_g2_two_chunks",
                                  "tc_g4_dense_pages"])
def test_chunked_prefill_debug_build(debug_build, name):
    P.test_chunked_prefill_matches_oracle(name)


@pytest.mark.parametrize("name", ["tiny_f32_c0", "bf16_g4", "bf16_short_ctx"])
def test_per_token_decode_debug_build(debug_build, name):
    P.test_per_token_decode_matches_oracle(name)


def test_buffered_decode_debug_build(debug_build):
    P.test_buffered_decode_matches_oracle()


@pytest.mark.parametrize("name", ["from_empty", "d64_g8"])
def test_attention_first_decode_debug_build(debug_build, name):
    P.test_attention_first_decode_step(name)


def test_compaction_debug_build(debug_build):
    P.test_compact_chunks_and_ring("bf16")


def test_rethreshold_debug_build(debug_build):
    RT.test_rethreshold_then_decode_matches_oracle("bf16_g4")


def test_sequence_split_debug_build(debug_build):
    SQ.test_split_decode_matches_oracle("g8_d64_three_slices")
