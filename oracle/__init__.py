"""Float64 CPU oracle of the SparseSAM hot path. Test infrastructure only: see sparsesam_oracle."""
