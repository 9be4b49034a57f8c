"""The TMA-staged warp-specialised kernel (gla_fwd_pipe) vs the fp64 oracle (GPU only).

The library selects it with GTR_KERNEL=pipe, for gtr_gla_fwd and gtr_gla_fwd_z.  The
parity, span, range and fused-gate tests of the default path run here again with that
selection: every workload and direction, the edge shapes (dk = 128 as two key halves),
dv = 128 (two value halves), degenerate gates, forced span counts (look-back and
corrections), in-place carry, split and resume, the large-key sub-block path, and the
gate formed from z at several temperatures and extreme pre-activations.
"""
import pytest

from tests.test_gpu_parity import (test_degenerate_gates, test_dv128_shapes, test_edge_shapes,  # noqa: F401
                                   test_empty_grid_copies_state, test_in_place_state_carry,
                                   test_large_sample_rows_match_oracle_subset,
                                   test_split_sequence_resume, test_workload_parity)
from tests.test_gpu_span import (test_forced_span_counts, test_in_place_carry_with_spans,  # noqa: F401
                                 test_long_spans_reread, test_ragged_last_span,
                                 test_span_groups_loop_over_sequences)
from tests.test_gpu_graph_range import (test_large_keys_take_the_sub_block_path_and_match,  # noqa: F401
                                        test_large_keys_with_spans_match, test_state_inside_fp16_is_exact)
from tests.test_gpu_gate_z import (test_dk128_with_fused_gate, test_temperatures_and_extreme_pre_activations,  # noqa: F401
                                   test_wide_values_with_fused_gate, test_workloads_with_fused_gate)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _pipe_kernel(monkeypatch):
    monkeypatch.setenv("GTR_KERNEL", "pipe")
