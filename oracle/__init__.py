"""Oracle package: plain fp64 CPU reference. Test infrastructure only."""
