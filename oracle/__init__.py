"""fp64 CPU oracle (test infrastructure only; see :mod:`oracle.dash_oracle`)."""
