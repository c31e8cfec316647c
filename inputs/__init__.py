from .gen import *  # noqa: F401,F403
from .gen import WORKLOADS, Workload, make_prefill, make_decode, make_decode_sequence, sample_rows, varlen_lengths  # noqa: F401
