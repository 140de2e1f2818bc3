"""Float64 CPU oracle (test infrastructure only; see ``hv_oracle``)."""
